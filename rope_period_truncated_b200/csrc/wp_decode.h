// Internal launch interface of the decode kernels (not part of the C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

namespace wp {

// Keys per split of the split-KV decode.
constexpr int DECODE_CHUNK = 1024;

struct DecodeArgs {
  const __nv_bfloat16 *q;            // [B, Hq, D]
  const __nv_bfloat16 *kc, *vc;      // V [B, Hkv, Lmax, D]; K the same or group-major [B, Hkv, D/16, Lmax, 16]
  const int32_t *lens;               // [B]
  __nv_bfloat16 *o;                  // [B, Hq, D]
  float *lse;                        // [B, Hq] or null
  float *o_part;                     // [B, Hq, nsplit, D]
  float *lse_part;                   // [B, Hq, nsplit], base-2
  int B, Hq, Hkv, Lmax, nsplit, chunk;
  int k_group_major;                 // K cache layout: 0 rows, 1 group-major (or windowed, below)
  int k_windowed;                    // K cache as per-group rings: group g of (b, hk) at
                                     // kc + (b * Hkv + hk) * wstride + wbase[g], key j in slot j % wcap[g]
  int32_t wcap[8];                   // ring capacity of each group (multiple of 16)
  int64_t wbase[8];                  // element offset of each group's ring
  int64_t wstride;                   // elements per (b, hk)
  const int32_t *block_table;        // paged cache: [B, max_pages] page of each page_size-key block, or null
  int max_pages, page_size, n_pages;
  int32_t cut[8];                    // group cutoffs (of the K loads: the union over heads / channels)
  float scale_log2;
  int mask;                          // DECODE_MASK_*: how scores are masked beyond the K loads
  int layout;                        // rotation layout (channel mode: which channel owns a dim)
};

// Score masking of the decode kernel. GROUP_SHARED: every head takes `cut`
// (the K loads already leave out-of-window groups as zeros). GROUP_PER_HEAD:
// query head h takes row h of a per-head table (the loads cover the union of
// the heads' windows and each head's scores are masked group by group).
// CHANNEL: the exact per-channel rule (one query position per sequence, so a
// channel's K dims are zeroed per key before the product). CHANNEL_PER_HEAD:
// the exact rule with one channel table per query head; the heads of a KV
// head share the K fragments, so each head's product takes the fragments
// masked by its own table (R products instead of one).
enum : int {
  DECODE_MASK_GROUP_SHARED = 0,
  DECODE_MASK_GROUP_PER_HEAD = 1,
  DECODE_MASK_CHANNEL = 2,
  DECODE_MASK_CHANNEL_PER_HEAD = 3
};

constexpr int DECODE_HEAD_CHAN_CAP = 2048;  // entries of the per-head channel table (H_q x D/2)

// Cutoff tables of the masked decode modes, a kernel parameter of their own.
struct DecodeTables {
  int32_t head_cut[1024];                         // [Hq][D/16] (GROUP_PER_HEAD)
  int32_t chan_cut[64];                           // [D/2] (CHANNEL)
  int32_t head_chan_cut[DECODE_HEAD_CHAN_CAP];  // [Hq][D/2] (CHANNEL_PER_HEAD)
};

// Scratch layout: o_part first, then lse_part at a 256-byte boundary.
inline size_t decode_partial_o_bytes(int B, int Hq, int nsplit, int D) {
  return (static_cast<size_t>(B) * Hq * nsplit * D * sizeof(float) + 255) & ~static_cast<size_t>(255);
}
inline size_t decode_workspace_bytes(int B, int Hq, int nsplit, int D) {
  return decode_partial_o_bytes(B, Hq, nsplit, D) +
         ((static_cast<size_t>(B) * Hq * nsplit * sizeof(float) + 255) & ~static_cast<size_t>(255));
}

cudaError_t launch_decode(const DecodeArgs &a, const DecodeTables *tables, int d_h, cudaStream_t stream);

// Ring capacities of the windowed K cache: group g keeps the last
// min(W_g + 1, Lmax) keys, rounded up to 16 (so a 16-key block aligned to 16
// never wraps). Returns the elements per (b, hk).
inline int64_t kcache_window_layout(const int32_t *cut, int G, int Lmax, int32_t *wcap, int64_t *wbase) {
  const int64_t lm = (static_cast<int64_t>(Lmax) + 15) / 16 * 16;
  int64_t off = 0;
  for (int g = 0; g < 8; ++g) {
    int64_t c = 0;
    if (g < G) {
      c = (static_cast<int64_t>(cut[g]) + 1 + 15) / 16 * 16;
      if (c > lm) c = lm;
    }
    wcap[g] = static_cast<int32_t>(c);
    wbase[g] = off;
    off += c * 16;
  }
  return off;
}

// Windowed K cache from rows: slot s of group g holds the latest key j < len
// with j % wcap[g] == s (zeros where there is none).
cudaError_t launch_kcache_window_from_rows(const __nv_bfloat16 *src, const int32_t *lens, __nv_bfloat16 *dst, int B,
                                           int Hkv, int Lmax, int D, const int32_t *wcap, const int64_t *wbase,
                                           int64_t wstride, cudaStream_t stream);
// Append one key per sequence (k_new [B, Hkv, D] at position pos[b]) into its rings.
cudaError_t launch_kcache_window_append(const __nv_bfloat16 *k_new, const int32_t *pos, __nv_bfloat16 *dst, int B,
                                        int Hkv, int Lmax, int D, const int32_t *wcap, const int64_t *wbase,
                                        int64_t wstride, cudaStream_t stream);

// K cache rows [BH, Lmax, D] -> group-major [BH, D/16, Lmax, 16] (BH = B * H_kv).
cudaError_t launch_kcache_group_major(const __nv_bfloat16 *src, __nv_bfloat16 *dst, int64_t BH, int Lmax, int D,
                                      cudaStream_t stream);

}  // namespace wp
