// Internal launch interface of the prefill kernels (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace wp {

// Entries of the cutoff tables carried in the kernel arguments: grouped mode
// takes cut_rows x d/16 entries, channel mode cut_rows x d/2.
constexpr int PREFILL_CUT_CAP = 2048;

// Where the rows of one sequence live. Uniform batch (cu_seqlens null):
// [B, N, H, d], sequence b at TMA coordinate (row, b) and output row
// b*N + i. Packed varlen batch: [T, H, d], sequence b at rows
// cu_seqlens[b] .. cu_seqlens[b+1]-1.
struct PrefillArgs {
  __nv_bfloat16 *o;           // [B, N, Hq, D] or [T, Hq, D]
  float *lse;                 // [B, Hq, N] or [Hq, T], or null
  int B, N, Hq, Hkv;          // N: length (uniform) or largest length (packed)
  int32_t cut[8];             // group cutoffs of every head (one table), D/16 entries
  float scale_log2;           // softmax scale * log2(e)
  long long wait_limit;
  const int32_t *cu_seqlens;  // device [B+1] or null
  int64_t T;                  // total tokens of a packed batch
  int cut_rows;               // 1: cut; Hq: HeadCuts, one row per query head
};

// Per-head group cutoffs [Hq][D/16], a kernel parameter of its own that only
// the per-head instantiations of the prefill kernel carry.
struct HeadCuts {
  int32_t cut[PREFILL_CUT_CAP];
};

struct ChannelPrefillArgs {
  const __nv_bfloat16 *q, *k, *v;  // [B, N, H, D] or [T, H, D]
  __nv_bfloat16 *o;
  float *lse;
  const int32_t *cu_seqlens;
  int B, N, Hq, Hkv, layout;
  int64_t T;
  int cut_rows;
  float scale_log2;
  long long wait_limit;          // bound of every mbarrier wait (tensor-core kernel)
  int32_t cut[PREFILL_CUT_CAP];  // [cut_rows][d/2] channel cutoffs
};

cudaError_t launch_prefill_grouped(int d_h, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                   const PrefillArgs &a, const HeadCuts *head_cuts, cudaStream_t stream);
cudaError_t launch_prefill_channel(int d_h, const ChannelPrefillArgs &a, cudaStream_t stream);

// Exact per-channel rule on the tensor cores (uniform and packed batches).
constexpr uint32_t PREFILL_SMEM_CAP = 232448;  // dynamic shared memory of one CTA
cudaError_t launch_prefill_exact(int d_h, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                 const ChannelPrefillArgs &a, cudaStream_t stream);

}  // namespace wp
