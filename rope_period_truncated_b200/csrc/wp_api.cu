// C ABI of libwaveprune.so: argument checks, cutoff tables, tile schedule,
// tensor maps and kernel launches. Declarations and contracts: waveprune.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "waveprune.h"
#include "wp_backward.h"
#include "wp_decode.h"
#include "wp_device.cuh"
#include "wp_prefill.h"
#include "wp_rope.h"
#include "wp_tile.h"

namespace wp {

__device__ int g_status = 0;

namespace {

constexpr long long DEFAULT_WAIT_LIMIT = 2000000000LL;  // SM cycles, about one second
long long g_wait_limit = DEFAULT_WAIT_LIMIT;

constexpr double kPi = 3.14159265358979323846;
constexpr double kLog2e = 1.4426950408889634074;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool head_dim_supported(int d_h) { return d_h == 64 || d_h == 128; }

// f_c = theta^(-2c/d_h) * freq_scale[c] * scale_all (WavePrune reading notes
// "WavePrune：RoPE 通常只需一个旋转周期", §1.1: the cutoffs follow the scaled
// frequencies).
double channel_freq(int c, int d_h, double theta, const double *freq_scale, double scale_all) {
  double f = std::pow(theta, -2.0 * static_cast<double>(c) / static_cast<double>(d_h));
  if (freq_scale != nullptr) f *= freq_scale[c];
  return f * scale_all;
}

bool freq_args_ok(int d_h, double theta, const double *freq_scale, double scale_all) {
  if (!(theta > 1.0) || !std::isfinite(theta)) return false;
  if (!(scale_all > 0.0) || !std::isfinite(scale_all)) return false;
  if (freq_scale != nullptr)
    for (int c = 0; c < d_h / 2; ++c)
      if (!(freq_scale[c] > 0.0) || !std::isfinite(freq_scale[c])) return false;
  return true;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 4-D bf16 view (d, H, N, B) of a [B, N, H, d] tensor; box (box_d, 1, box_rows, 1).
bool make_map(CUtensorMap *m, const void *base, int B, int N, int H, int d, int box_d, CUtensorMapSwizzle sw,
              int box_rows = 128) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H) * d * 2,
                           static_cast<cuuint64_t>(N) * H * d * 2};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(box_d), 1, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? WP_OK : WP_ERR_CUDA; }

__global__ void wait_probe_kernel(long long limit) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, limit, nullptr);  // nothing arrives: gives up after `limit`
  __syncthreads();
}

}  // namespace
}  // namespace wp

using namespace wp;

extern "C" {

int wp_cutoffs(int d_h, double theta, const double *freq_scale, double scale_all, double alpha, int layout,
               int32_t *chan_cut, int32_t *group_cut) {
  if (d_h < 16 || d_h % 16 != 0 || d_h > 1024) return WP_ERR_ARG;
  if (layout != WP_ROPE_INTERLEAVED && layout != WP_ROPE_HALF_SPLIT) return WP_ERR_ARG;
  if (!freq_args_ok(d_h, theta, freq_scale, scale_all) || !(alpha > 0.0)) return WP_ERR_ARG;
  const int C = d_h / 2;
  int32_t wc[512];
  // WavePrune reading notes, §2.1 (after Eq. (6)): w_c = alpha*pi/f_c, and a
  // channel is kept iff distance <= floor(w_c).
  for (int c = 0; c < C; ++c) {
    const double w = alpha * kPi / channel_freq(c, d_h, theta, freq_scale, scale_all);
    const double fl = std::floor(w);
    wc[c] = fl < 2147483647.0 ? static_cast<int32_t>(fl) : WP_CUTOFF_INF;
  }
  if (chan_cut != nullptr) std::memcpy(chan_cut, wc, sizeof(int32_t) * C);
  // §2.3 Eq. (8): the group cutoff is the largest cutoff of the channels that
  // own its 16 dims (interleaved: dim k -> channel k/2; half-split: k mod C).
  if (group_cut != nullptr)
    for (int g = 0; g < d_h / 16; ++g) {
      int32_t m = 0;
      for (int k = 16 * g; k < 16 * g + 16; ++k) {
        const int c = layout == WP_ROPE_INTERLEAVED ? k / 2 : k % C;
        if (wc[c] > m) m = wc[c];
      }
      group_cut[g] = m;
    }
  return WP_OK;
}

int wp_schedule(int N, int BM, int BN, const int32_t *cut, int n_cut, uint8_t *cls, int64_t *counts) {
  if (N <= 0 || BM <= 0 || BN <= 0 || cut == nullptr || counts == nullptr || n_cut < 1 || n_cut > 64)
    return WP_ERR_ARG;
  for (int g = 0; g < n_cut; ++g)
    if (cut[g] < 0) return WP_ERR_ARG;
  const int64_t nqb = (static_cast<int64_t>(N) + BM - 1) / BM, nkb = (static_cast<int64_t>(N) + BN - 1) / BN;
  for (int g = 0; g < 3 * n_cut; ++g) counts[g] = 0;
  for (int64_t qb = 0; qb < nqb; ++qb)
    for (int64_t kb = 0; kb < nkb; ++kb) {
      int64_t dmin = 0, dmax = -1;
      const bool causal = tile_distance_range(N, BM, BN, qb, kb, &dmin, &dmax);
      for (int g = 0; g < n_cut; ++g) {
        const int c = causal ? classify_cutoff(dmin, dmax, cut[g]) : TILE_NONE;
        if (cls != nullptr) cls[(qb * nkb + kb) * n_cut + g] = static_cast<uint8_t>(c);
        if (c != TILE_NONE) counts[3 * g + c] += 1;
      }
    }
  return WP_OK;
}

int wp_rope_apply(const void *x, void *y, int B, int N, int H, int d_h, const int32_t *pos, int pos0, double theta,
                  const double *freq_scale, double scale_all, int layout, void *stream) {
  if (x == nullptr || y == nullptr || !aligned16(x) || !aligned16(y)) return WP_ERR_ARG;
  if (B <= 0 || N <= 0 || H <= 0) return WP_ERR_ARG;
  if (layout != WP_ROPE_INTERLEAVED && layout != WP_ROPE_HALF_SPLIT && layout != WP_ROPE_HALF_SPLIT_PAIRED)
    return WP_ERR_ARG;
  if (!head_dim_supported(d_h)) return d_h > 0 && d_h % 16 == 0 ? WP_ERR_UNSUPPORTED : WP_ERR_ARG;
  if (!freq_args_ok(d_h, theta, freq_scale, scale_all)) return WP_ERR_ARG;
  if (layout == WP_ROPE_HALF_SPLIT_PAIRED && x == y) return WP_ERR_ARG;  // permutes dims: not in place
  if (x != y) {  // only exact in-place aliasing is allowed
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(x), b0 = reinterpret_cast<uintptr_t>(y);
    const uintptr_t n = static_cast<uintptr_t>(B) * N * H * d_h * 2;
    if (a0 < b0 + n && b0 < a0 + n) return WP_ERR_ARG;
  }
  RopeArgs a;
  a.x = static_cast<const __nv_bfloat16 *>(x);
  a.y = static_cast<__nv_bfloat16 *>(y);
  a.pos = pos;
  a.tokens = static_cast<int64_t>(B) * N;
  a.N = N;
  a.H = H;
  a.pos0 = pos0;
  for (int c = 0; c < 64; ++c) a.freq[c] = c < d_h / 2 ? channel_freq(c, d_h, theta, freq_scale, scale_all) : 0.0;
  return from_cuda(launch_rope(a, d_h, layout, static_cast<cudaStream_t>(stream)));
}

int wp_prefill_ex(const void *q, const void *k, const void *v, void *o, float *lse, const int32_t *cu_seqlens,
                  int B, int N, int64_t total_tokens, int H_q, int H_kv, int d_h, int mode, const int32_t *cut,
                  int cut_rows, int layout, float softmax_scale, void *stream) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return WP_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse != nullptr && !aligned16(lse)))
    return WP_ERR_ARG;
  if (B <= 0 || N <= 0 || H_q <= 0 || H_kv <= 0 || H_q % H_kv != 0) return WP_ERR_ARG;
  if (cu_seqlens != nullptr && ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0 || total_tokens <= 0))
    return WP_ERR_ARG;
  if (B > 65535 || H_q > 65535) return WP_ERR_UNSUPPORTED;
  if (mode != WP_MODE_GROUPED && mode != WP_MODE_CHANNEL) return WP_ERR_ARG;
  if (layout != WP_ROPE_INTERLEAVED && layout != WP_ROPE_HALF_SPLIT) return WP_ERR_ARG;
  if (!head_dim_supported(d_h)) return d_h > 0 && d_h % 16 == 0 ? WP_ERR_UNSUPPORTED : WP_ERR_ARG;
  if (!std::isfinite(softmax_scale)) return WP_ERR_ARG;
  if (cut_rows != 1 && cut_rows != H_q) return WP_ERR_ARG;
  if (cut_rows != 1 && cut == nullptr) return WP_ERR_ARG;
  // the packed view is [T, H, d]: row coordinates of the tensor maps are int32
  if (cu_seqlens != nullptr && total_tokens > (1ll << 31) - 256) return WP_ERR_UNSUPPORTED;
  const int per_row = mode == WP_MODE_GROUPED ? d_h / 16 : d_h / 2;
  if (static_cast<int64_t>(cut_rows) * per_row > PREFILL_CUT_CAP) return WP_ERR_UNSUPPORTED;
  const float scale = softmax_scale > 0.f ? softmax_scale : static_cast<float>(1.0 / std::sqrt(double(d_h)));
  const float scale_log2 = static_cast<float>(static_cast<double>(scale) * kLog2e);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t T = cu_seqlens != nullptr ? total_tokens : static_cast<int64_t>(B) * N;

  if (mode == WP_MODE_CHANNEL) {
    ChannelPrefillArgs a;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.k = static_cast<const __nv_bfloat16 *>(k);
    a.v = static_cast<const __nv_bfloat16 *>(v);
    a.o = static_cast<__nv_bfloat16 *>(o);
    a.lse = lse;
    a.cu_seqlens = cu_seqlens;
    a.B = B;
    a.N = N;
    a.T = T;
    a.Hq = H_q;
    a.Hkv = H_kv;
    a.layout = layout;
    a.cut_rows = cut_rows;
    for (int e = 0; e < cut_rows * per_row; ++e) {
      a.cut[e] = cut == nullptr ? WP_CUTOFF_INF : cut[e];
      if (a.cut[e] < 0) return WP_ERR_ARG;
    }
    a.scale_log2 = scale_log2;
    a.wait_limit = g_wait_limit;
    // the tensor-core kernel (uniform and packed batches) within its grid limits,
    // else the CUDA-core kernel
    if ((N + 127) / 128 <= 65535 && static_cast<int64_t>(H_kv) * B <= 65535) {
      const int mB = cu_seqlens != nullptr ? 1 : B;
      const int mN = cu_seqlens != nullptr ? static_cast<int>(total_tokens) : N;
      CUtensorMap tq, tk, tv;
      if (!make_map(&tq, q, mB, mN, H_q, d_h, 16, CU_TENSOR_MAP_SWIZZLE_32B) ||
          !make_map(&tk, k, mB, mN, H_kv, d_h, 16, CU_TENSOR_MAP_SWIZZLE_32B) ||
          !make_map(&tv, v, mB, mN, H_kv, d_h, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return WP_ERR_CUDA;
      return from_cuda(launch_prefill_exact(d_h, tq, tk, tv, a, s));
    }
    return from_cuda(launch_prefill_channel(d_h, a, s));
  }

  if ((N + 127) / 128 > 65535 || static_cast<int64_t>(H_kv) * B > 65535) return WP_ERR_UNSUPPORTED;
  // the kernel keeps one key-block table per CTA in shared memory: 2^20 tokens fit at every d_h
  if (N > (1 << 20)) return WP_ERR_UNSUPPORTED;
  // with one table per head, two tables share that space: 2^19 tokens
  if (cut_rows != 1 && N > (1 << 19)) return WP_ERR_UNSUPPORTED;
  PrefillArgs a;
  a.o = static_cast<__nv_bfloat16 *>(o);
  a.lse = lse;
  a.cu_seqlens = cu_seqlens;
  a.B = B;
  a.N = N;
  a.T = T;
  a.Hq = H_q;
  a.Hkv = H_kv;
  a.cut_rows = cut_rows;
  for (int g = 0; g < 8; ++g) a.cut[g] = WP_CUTOFF_INF;
  HeadCuts hc;
  for (int e = 0; e < cut_rows * per_row; ++e) {
    const int32_t w = cut == nullptr ? WP_CUTOFF_INF : cut[e];
    if (w < 0) return WP_ERR_ARG;
    if (cut_rows == 1)
      a.cut[e] = w;
    else
      hc.cut[e] = w;
  }
  a.scale_log2 = scale_log2;
  a.wait_limit = g_wait_limit;
  CUtensorMap tq, tk, tv;
  const int mB = cu_seqlens != nullptr ? 1 : B;
  const int mN = cu_seqlens != nullptr ? static_cast<int>(total_tokens) : N;
  if (!make_map(&tq, q, mB, mN, H_q, d_h, 16, CU_TENSOR_MAP_SWIZZLE_32B) ||
      !make_map(&tk, k, mB, mN, H_kv, d_h, 16, CU_TENSOR_MAP_SWIZZLE_32B) ||
      !make_map(&tv, v, mB, mN, H_kv, d_h, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return WP_ERR_CUDA;
  return from_cuda(launch_prefill_grouped(d_h, tq, tk, tv, a, cut_rows == 1 ? nullptr : &hc, s));
}

int wp_prefill(const void *q, const void *k, const void *v, void *o, float *lse, int B, int N, int H_q, int H_kv,
               int d_h, int mode, const int32_t *cut, int layout, float softmax_scale, void *stream) {
  return wp_prefill_ex(q, k, v, o, lse, nullptr, B, N, 0, H_q, H_kv, d_h, mode, cut, 1, layout, softmax_scale,
                       stream);
}

size_t wp_prefill_backward_workspace_bytes(int B, int N, int H_q) {
  if (B <= 0 || N <= 0 || H_q <= 0) return 0;
  return (static_cast<size_t>(B) * H_q * N * sizeof(float) + 255) & ~static_cast<size_t>(255);
}

int wp_prefill_backward(const void *q, const void *k, const void *v, const void *o, const void *dout, const float *lse,
                        void *dq, void *dk, void *dv, void *workspace, size_t ws_bytes, int B, int N, int H_q,
                        int H_kv, int d_h, const int32_t *cut, int cut_rows, float softmax_scale, void *stream) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || dout == nullptr || lse == nullptr ||
      dq == nullptr || dk == nullptr || dv == nullptr || workspace == nullptr)
    return WP_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return WP_ERR_ARG;
  if (B <= 0 || N <= 0 || H_q <= 0 || H_kv <= 0 || H_q % H_kv != 0) return WP_ERR_ARG;
  if (!head_dim_supported(d_h)) return d_h > 0 && d_h % 16 == 0 ? WP_ERR_UNSUPPORTED : WP_ERR_ARG;
  if (B > 65535 || H_q > 65535 || H_kv > 65535) return WP_ERR_UNSUPPORTED;
  if (!std::isfinite(softmax_scale)) return WP_ERR_ARG;
  if (cut_rows != 1 && cut_rows != H_q) return WP_ERR_ARG;
  if (cut_rows != 1 && cut == nullptr) return WP_ERR_ARG;
  if (ws_bytes < wp_prefill_backward_workspace_bytes(B, N, H_q)) return WP_ERR_ARG;
  const int G = d_h / 16;
  if (static_cast<int64_t>(cut_rows) * G > PREFILL_CUT_CAP) return WP_ERR_UNSUPPORTED;
  // the key-major kernel keeps the cutoff rows of the query heads of one KV head in shared memory
  if (H_q / H_kv > 64) return WP_ERR_UNSUPPORTED;
  const float scale = softmax_scale > 0.f ? softmax_scale : static_cast<float>(1.0 / std::sqrt(double(d_h)));
  BackwardArgs a;
  a.q = static_cast<const __nv_bfloat16 *>(q);
  a.k = static_cast<const __nv_bfloat16 *>(k);
  a.v = static_cast<const __nv_bfloat16 *>(v);
  a.o = static_cast<const __nv_bfloat16 *>(o);
  a.dout = static_cast<const __nv_bfloat16 *>(dout);
  a.lse = lse;
  a.delta = static_cast<float *>(workspace);
  a.dq = static_cast<__nv_bfloat16 *>(dq);
  a.dk = static_cast<__nv_bfloat16 *>(dk);
  a.dv = static_cast<__nv_bfloat16 *>(dv);
  a.B = B;
  a.N = N;
  a.Hq = H_q;
  a.Hkv = H_kv;
  a.cut_rows = cut_rows;
  for (int e = 0; e < cut_rows * G; ++e) {
    a.cut[e] = cut == nullptr ? WP_CUTOFF_INF : cut[e];
    if (a.cut[e] < 0) return WP_ERR_ARG;
  }
  a.scale = scale;
  a.scale_log2 = static_cast<float>(static_cast<double>(scale) * kLog2e);
  a.wait_limit = g_wait_limit;
  if ((N + 127) / 128 > 65535) return WP_ERR_UNSUPPORTED;
  BackwardMaps m;
  const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_32B;
  if (!make_map(&m.q128, q, B, N, H_q, d_h, 16, sw, 128) || !make_map(&m.do128, dout, B, N, H_q, d_h, 16, sw, 128) ||
      !make_map(&m.k64, k, B, N, H_kv, d_h, 16, sw, 64) || !make_map(&m.v64, v, B, N, H_kv, d_h, 16, sw, 64) ||
      !make_map(&m.k128, k, B, N, H_kv, d_h, 16, sw, 128) || !make_map(&m.v128, v, B, N, H_kv, d_h, 16, sw, 128) ||
      !make_map(&m.q64, q, B, N, H_q, d_h, 16, sw, 64) || !make_map(&m.do64, dout, B, N, H_q, d_h, 16, sw, 64))
    return WP_ERR_CUDA;
  return from_cuda(launch_backward(d_h, a, m, static_cast<cudaStream_t>(stream)));
}

size_t wp_decode_workspace_bytes(int B, int H_q, int d_h, int Lmax) {
  if (B <= 0 || H_q <= 0 || d_h <= 0 || Lmax <= 0) return 0;
  const int nsplit = (Lmax + DECODE_CHUNK - 1) / DECODE_CHUNK;
  return decode_workspace_bytes(B, H_q, nsplit, d_h);
}

// Shared argument checks and launch of the split-KV decode; block_table null
// = contiguous caches of Lmax keys, else pages of page_size keys.
// mask / tables: DECODE_MASK_GROUP_SHARED with group_cut (NULL: dense), or a
// masked mode with its tables, group_cut then holding the loads' cutoffs.
static int decode_launch(const void *q, const void *kcache, int k_layout, const void *vcache, const int32_t *lens,
                         int Lmax, int B, int H_q, int H_kv, int d_h, const int32_t *group_cut, float softmax_scale,
                         void *o, float *lse, void *workspace, size_t ws_bytes, const int32_t *block_table,
                         int max_pages, int page_size, int n_pages, void *stream, int mask = DECODE_MASK_GROUP_SHARED,
                         int layout = WP_ROPE_INTERLEAVED, const DecodeTables *tables = nullptr) {
  if (q == nullptr || kcache == nullptr || vcache == nullptr || lens == nullptr || o == nullptr ||
      workspace == nullptr)
    return WP_ERR_ARG;
  if (k_layout != WP_KCACHE_ROWS && k_layout != WP_KCACHE_GROUP_MAJOR && k_layout != WP_KCACHE_WINDOWED)
    return WP_ERR_ARG;
  // the windowed rings follow the group cutoffs of a plain grouped decode
  if (k_layout == WP_KCACHE_WINDOWED &&
      (group_cut == nullptr || block_table != nullptr || mask != DECODE_MASK_GROUP_SHARED))
    return group_cut == nullptr ? WP_ERR_ARG : WP_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || (reinterpret_cast<uintptr_t>(lens) & 3u) != 0 ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0))
    return WP_ERR_ARG;
  if (B <= 0 || Lmax <= 0 || H_q <= 0 || H_kv <= 0 || H_q % H_kv != 0) return WP_ERR_ARG;
  if (!head_dim_supported(d_h)) return d_h > 0 && d_h % 16 == 0 ? WP_ERR_UNSUPPORTED : WP_ERR_ARG;
  const int R = H_q / H_kv;
  if (R != 1 && R != 2 && R != 4 && R != 8) return WP_ERR_UNSUPPORTED;
  if (B > 65535 || H_kv > 65535) return WP_ERR_UNSUPPORTED;
  if (!std::isfinite(softmax_scale)) return WP_ERR_ARG;
  const int nsplit = (Lmax + DECODE_CHUNK - 1) / DECODE_CHUNK;
  if (ws_bytes < decode_workspace_bytes(B, H_q, nsplit, d_h)) return WP_ERR_ARG;
  const float scale = softmax_scale > 0.f ? softmax_scale : static_cast<float>(1.0 / std::sqrt(double(d_h)));
  DecodeArgs a;
  a.q = static_cast<const __nv_bfloat16 *>(q);
  a.kc = static_cast<const __nv_bfloat16 *>(kcache);
  a.vc = static_cast<const __nv_bfloat16 *>(vcache);
  a.lens = lens;
  a.o = static_cast<__nv_bfloat16 *>(o);
  a.lse = lse;
  a.o_part = static_cast<float *>(workspace);
  a.lse_part = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) +
                                         decode_partial_o_bytes(B, H_q, nsplit, d_h));
  a.B = B;
  a.Hq = H_q;
  a.Hkv = H_kv;
  a.Lmax = Lmax;
  a.nsplit = nsplit;
  a.chunk = DECODE_CHUNK;
  a.k_group_major = k_layout != WP_KCACHE_ROWS ? 1 : 0;
  a.k_windowed = k_layout == WP_KCACHE_WINDOWED ? 1 : 0;
  a.block_table = block_table;
  a.max_pages = max_pages;
  a.page_size = page_size;
  a.n_pages = n_pages;
  for (int g = 0; g < 8; ++g) {
    a.cut[g] = (group_cut == nullptr || g >= d_h / 16) ? WP_CUTOFF_INF : group_cut[g];
    if (a.cut[g] < 0) return WP_ERR_ARG;
  }
  a.wstride = a.k_windowed ? kcache_window_layout(a.cut, d_h / 16, Lmax, a.wcap, a.wbase) : 0;
  if (!a.k_windowed)
    for (int g = 0; g < 8; ++g) {
      a.wcap[g] = 0;
      a.wbase[g] = 0;
    }
  a.scale_log2 = static_cast<float>(static_cast<double>(scale) * kLog2e);
  a.mask = mask;
  a.layout = layout;
  return from_cuda(launch_decode(a, tables, d_h, static_cast<cudaStream_t>(stream)));
}

int wp_decode_kl(const void *q, const void *kcache, int k_layout, const void *vcache, const int32_t *lens, int Lmax,
                 int B, int H_q, int H_kv, int d_h, const int32_t *group_cut, float softmax_scale, void *o, float *lse,
                 void *workspace, size_t ws_bytes, void *stream) {
  return decode_launch(q, kcache, k_layout, vcache, lens, Lmax, B, H_q, H_kv, d_h, group_cut, softmax_scale, o, lse,
                       workspace, ws_bytes, nullptr, 0, 0, 0, stream);
}

int wp_decode_ex(const void *q, const void *kcache, int k_layout, const void *vcache, const int32_t *lens, int Lmax,
                 int B, int H_q, int H_kv, int d_h, int mode, const int32_t *cut, int cut_rows, int layout,
                 float softmax_scale, void *o, float *lse, void *workspace, size_t ws_bytes, void *stream) {
  if (mode != WP_MODE_GROUPED && mode != WP_MODE_CHANNEL) return WP_ERR_ARG;
  if (layout != WP_ROPE_INTERLEAVED && layout != WP_ROPE_HALF_SPLIT) return WP_ERR_ARG;
  if (H_q <= 0 || (cut_rows != 1 && cut_rows != H_q)) return WP_ERR_ARG;
  if (cut_rows != 1 && cut == nullptr) return WP_ERR_ARG;
  if (!head_dim_supported(d_h)) return d_h > 0 && d_h % 16 == 0 ? WP_ERR_UNSUPPORTED : WP_ERR_ARG;
  const int G = d_h / 16, C = d_h / 2;
  if (mode == WP_MODE_GROUPED && cut_rows == 1)
    return decode_launch(q, kcache, k_layout, vcache, lens, Lmax, B, H_q, H_kv, d_h, cut, softmax_scale, o, lse,
                         workspace, ws_bytes, nullptr, 0, 0, 0, stream);
  if (mode == WP_MODE_CHANNEL && cut_rows != 1 && static_cast<int64_t>(H_q) * C > DECODE_HEAD_CHAN_CAP)
    return WP_ERR_UNSUPPORTED;
  DecodeTables tables;
  int32_t load_cut[8];
  if (mode == WP_MODE_CHANNEL && cut_rows != 1) {
    // exact rule, one channel row per query head: a group's K loads follow the
    // largest cutoff of its channels over all heads
    for (int e = 0; e < H_q * C; ++e) {
      if (cut[e] < 0) return WP_ERR_ARG;
      tables.head_chan_cut[e] = cut[e];
    }
    for (int g = 0; g < G; ++g) {
      int32_t m = 0;
      for (int h = 0; h < H_q; ++h)
        for (int k = 16 * g; k < 16 * g + 16; ++k) {
          const int c = layout == WP_ROPE_INTERLEAVED ? k / 2 : k % C;
          m = tables.head_chan_cut[h * C + c] > m ? tables.head_chan_cut[h * C + c] : m;
        }
      load_cut[g] = m;
    }
    return decode_launch(q, kcache, k_layout, vcache, lens, Lmax, B, H_q, H_kv, d_h, load_cut, softmax_scale, o,
                         lse, workspace, ws_bytes, nullptr, 0, 0, 0, stream, DECODE_MASK_CHANNEL_PER_HEAD, layout,
                         &tables);
  }
  if (mode == WP_MODE_GROUPED) {
    if (static_cast<int64_t>(H_q) * G > 1024) return WP_ERR_UNSUPPORTED;
    // the K loads cover the union of the heads' windows
    for (int g = 0; g < G; ++g) load_cut[g] = 0;
    for (int e = 0; e < H_q * G; ++e) {
      if (cut[e] < 0) return WP_ERR_ARG;
      tables.head_cut[e] = cut[e];
      load_cut[e % G] = cut[e] > load_cut[e % G] ? cut[e] : load_cut[e % G];
    }
  } else {
    // exact rule: a group's K loads follow its largest channel cutoff
    for (int c = 0; c < C; ++c) {
      tables.chan_cut[c] = cut == nullptr ? WP_CUTOFF_INF : cut[c];
      if (tables.chan_cut[c] < 0) return WP_ERR_ARG;
    }
    for (int g = 0; g < G; ++g) {
      int32_t m = 0;
      for (int k = 16 * g; k < 16 * g + 16; ++k) {
        const int c = layout == WP_ROPE_INTERLEAVED ? k / 2 : k % C;
        m = tables.chan_cut[c] > m ? tables.chan_cut[c] : m;
      }
      load_cut[g] = m;
    }
  }
  return decode_launch(q, kcache, k_layout, vcache, lens, Lmax, B, H_q, H_kv, d_h, load_cut, softmax_scale, o, lse,
                       workspace, ws_bytes, nullptr, 0, 0, 0, stream,
                       mode == WP_MODE_GROUPED ? DECODE_MASK_GROUP_PER_HEAD : DECODE_MASK_CHANNEL, layout, &tables);
}

int wp_decode_paged(const void *q, const void *k_pages, int k_layout, const void *v_pages, int n_pages, int page_size,
                    const int32_t *block_table, int max_pages, const int32_t *lens, int B, int H_q, int H_kv, int d_h,
                    const int32_t *group_cut, float softmax_scale, void *o, float *lse, void *workspace,
                    size_t ws_bytes, void *stream) {
  if (block_table == nullptr || (reinterpret_cast<uintptr_t>(block_table) & 3u) != 0) return WP_ERR_ARG;
  if (n_pages <= 0 || max_pages <= 0 || page_size < 16 || page_size % 16 != 0) return WP_ERR_ARG;
  const int64_t Lmax = static_cast<int64_t>(max_pages) * page_size;
  if (Lmax > (1ll << 30)) return WP_ERR_UNSUPPORTED;
  return decode_launch(q, k_pages, k_layout, v_pages, lens, static_cast<int>(Lmax), B, H_q, H_kv, d_h, group_cut,
                       softmax_scale, o, lse, workspace, ws_bytes, block_table, max_pages, page_size, n_pages, stream);
}

int wp_decode(const void *q, const void *kcache, const void *vcache, const int32_t *lens, int Lmax, int B, int H_q,
              int H_kv, int d_h, const int32_t *group_cut, float softmax_scale, void *o, float *lse,
              void *workspace, size_t ws_bytes, void *stream) {
  return wp_decode_kl(q, kcache, WP_KCACHE_ROWS, vcache, lens, Lmax, B, H_q, H_kv, d_h, group_cut, softmax_scale, o,
                      lse, workspace, ws_bytes, stream);
}

// Checks shared by the windowed-cache calls; fills the ring geometry.
static int window_args(int B, int H_kv, int Lmax, int d_h, const int32_t *group_cut, int32_t *wcap, int64_t *wbase,
                       int64_t *wstride) {
  if (B <= 0 || H_kv <= 0 || Lmax <= 0 || group_cut == nullptr) return WP_ERR_ARG;
  if (!head_dim_supported(d_h)) return d_h > 0 && d_h % 16 == 0 ? WP_ERR_UNSUPPORTED : WP_ERR_ARG;
  int32_t cut[8];
  for (int g = 0; g < 8; ++g) {
    cut[g] = g < d_h / 16 ? group_cut[g] : 0;
    if (cut[g] < 0) return WP_ERR_ARG;
  }
  *wstride = kcache_window_layout(cut, d_h / 16, Lmax, wcap, wbase);
  return WP_OK;
}
size_t wp_kcache_windowed_elems(int Lmax, int d_h, const int32_t *group_cut) {
  int32_t wcap[8];
  int64_t wbase[8], wstride = 0;
  if (window_args(1, 1, Lmax, d_h, group_cut, wcap, wbase, &wstride) != WP_OK) return 0;
  return static_cast<size_t>(wstride);
}
int wp_kcache_windowed_from_rows(const void *k_rows, const int32_t *lens, void *k_win, int B, int H_kv, int Lmax,
                                 int d_h, const int32_t *group_cut, void *stream) {
  if (k_rows == nullptr || lens == nullptr || k_win == nullptr || !aligned16(k_rows) || !aligned16(k_win) ||
      (reinterpret_cast<uintptr_t>(lens) & 3u) != 0 || k_rows == k_win)
    return WP_ERR_ARG;
  int32_t wcap[8];
  int64_t wbase[8], wstride = 0;
  const int rc = window_args(B, H_kv, Lmax, d_h, group_cut, wcap, wbase, &wstride);
  if (rc != WP_OK) return rc;
  return from_cuda(launch_kcache_window_from_rows(static_cast<const __nv_bfloat16 *>(k_rows), lens,
                                                  static_cast<__nv_bfloat16 *>(k_win), B, H_kv, Lmax, d_h, wcap,
                                                  wbase, wstride, static_cast<cudaStream_t>(stream)));
}
int wp_kcache_windowed_append(const void *k_new, const int32_t *pos, void *k_win, int B, int H_kv, int Lmax, int d_h,
                              const int32_t *group_cut, void *stream) {
  if (k_new == nullptr || pos == nullptr || k_win == nullptr || !aligned16(k_new) || !aligned16(k_win) ||
      (reinterpret_cast<uintptr_t>(pos) & 3u) != 0)
    return WP_ERR_ARG;
  int32_t wcap[8];
  int64_t wbase[8], wstride = 0;
  const int rc = window_args(B, H_kv, Lmax, d_h, group_cut, wcap, wbase, &wstride);
  if (rc != WP_OK) return rc;
  return from_cuda(launch_kcache_window_append(static_cast<const __nv_bfloat16 *>(k_new), pos,
                                               static_cast<__nv_bfloat16 *>(k_win), B, H_kv, Lmax, d_h, wcap, wbase,
                                               wstride, static_cast<cudaStream_t>(stream)));
}

int wp_kcache_group_major(const void *k_rows, void *k_gm, int B, int H_kv, int Lmax, int d_h, void *stream) {
  if (k_rows == nullptr || k_gm == nullptr || !aligned16(k_rows) || !aligned16(k_gm)) return WP_ERR_ARG;
  if (B <= 0 || H_kv <= 0 || Lmax <= 0) return WP_ERR_ARG;
  if (!head_dim_supported(d_h)) return d_h > 0 && d_h % 16 == 0 ? WP_ERR_UNSUPPORTED : WP_ERR_ARG;
  if (k_rows == k_gm) return WP_ERR_ARG;  // not in place
  return from_cuda(launch_kcache_group_major(static_cast<const __nv_bfloat16 *>(k_rows),
                                             static_cast<__nv_bfloat16 *>(k_gm), static_cast<int64_t>(B) * H_kv,
                                             Lmax, d_h, static_cast<cudaStream_t>(stream)));
}

int wp_device_status(void *stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return WP_ERR_CUDA;
  int h = 0;
  if (cudaMemcpyFromSymbol(&h, g_status, sizeof(int)) != cudaSuccess) return WP_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return WP_ERR_CUDA;
  return h == 0 ? WP_OK : h;
}

long long wp_set_wait_limit(long long cycles) {
  const long long prev = g_wait_limit;
  g_wait_limit = cycles > 0 ? cycles : DEFAULT_WAIT_LIMIT;
  return prev;
}

int wp_wait_probe(void *stream) {
  wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(g_wait_limit);
  return from_cuda(cudaGetLastError());
}

const char *wp_status_str(int status) {
  switch (status) {
    case WP_OK: return "ok";
    case WP_ERR_ARG: return "invalid argument";
    case WP_ERR_UNSUPPORTED: return "unsupported configuration";
    case WP_ERR_CUDA: return "CUDA error";
    case WP_ERR_TIMEOUT: return "kernel gave up waiting on an internal barrier";
    default: return "unknown status";
  }
}

}  // extern "C"
