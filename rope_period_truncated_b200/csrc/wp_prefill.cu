// WavePrune grouped-cutoff causal prefill on sm_100a: TMA + tcgen05 + TMEM.
//
// What it computes (WavePrune reading notes "WavePrune：RoPE 通常只需一个旋转
// 周期", §2.1 Eq. (6) and §2.3 Eq. (8)): for j <= i,
//   L_ij = scale * sum_g 1[i - j <= W_g] * (Q_i[16g:16g+16] . K_j[16g:16g+16]),
// then the usual causal softmax and O = A V. A masked group adds 0 to the
// logit (detail 1 of §2.1), the pair stays in the softmax.
//
// How (one CTA per 128-row query tile of one query head, key tiles of 128
// visited from the diagonal backwards):
//   warp 4  TMA producer: Q once (one 16-dim box per group); per key tile only
//           the K column slices of non-skipped groups (16-dim boxes, 32-byte
//           swizzle) and all of V (64-dim boxes, 128-byte swizzle).
//   warp 5  MMA issuer: per key tile one tcgen05.mma (M=128, N=128, K=16) per
//           non-skipped group; full groups accumulate into S_full (TMEM),
//           boundary groups into the separate S_bnd accumulator, one distinct
//           cutoff at a time in ascending order. Then P (bf16, written back
//           into TMEM by the softmax warps) times V into the O accumulator.
//   warps 0-3  one thread per query row: read S_full, add each boundary
//           accumulator under its per-element mask, causal mask on the
//           diagonal tile, online softmax (base-2, scale folded in), write P
//           to TMEM, rescale O when the row max grows; epilogue O/l -> bf16,
//           LSE = ln(sum exp).
// TMEM columns: [0, D) O, [128, 256) S_full buffer 0, [256, 384) buffer 1,
// [384, 512) S_bnd. S_full is double-buffered so the QK MMAs of the next key
// tile overlap the softmax of the current one.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "wp_device.cuh"
#include "wp_prefill.h"
#include "wp_tile.h"

namespace wp {

namespace {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int KST = 3;  // K stages
constexpr int VST = 2;  // V stages
constexpr int NTHREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_O = 0;
constexpr uint32_t COL_S0 = 128;
constexpr uint32_t COL_SB = 384;
constexpr uint32_t GROUP_TILE_BYTES = 128 * 32;     // 128 rows x 16 bf16
constexpr uint32_t V_CHUNK_BYTES = 128 * 128;       // 128 keys x 64 bf16

template <int D>
struct Layout {
  static constexpr int G = D / 16;
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t K_OFF = Q_OFF + G * GROUP_TILE_BYTES;
  static constexpr uint32_t K_STAGE = G * GROUP_TILE_BYTES;
  static constexpr uint32_t V_OFF = K_OFF + KST * K_STAGE;
  static constexpr uint32_t V_STAGE = (D / 64) * V_CHUNK_BYTES;
  static constexpr uint32_t BAR_OFF = V_OFF + VST * V_STAGE;
  static constexpr uint32_t NUM_BARS = 1 + 2 * KST + 2 * VST + 2 + 2 + 2 + 1 + 1;
  static constexpr uint32_t MISC_OFF = BAR_OFF + NUM_BARS * 8;
  static constexpr uint32_t BYTES = MISC_OFF + 16;
  static constexpr uint32_t ALLOC = BYTES + 1024;  // slack for 1024-byte alignment
};

struct Barriers {
  uint64_t *q_full, *k_full, *k_empty, *v_full, *v_empty, *s_ready, *bnd_ready, *bnd_free, *p_ready, *o_ready,
      *drain;
};

// Row-max growth (base-2 units) below which O is not rescaled.
constexpr float RESCALE_THRESHOLD = 8.0f;

// All lanes poll the barrier, then the warp agrees: the result is uniform and
// the warp is converged for the .sync.aligned TMEM instructions that follow.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, long long lim, volatile int *abort_flag) {
  const bool ok = mbar_wait(bar, parity, lim, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

// Per key tile: groups computed without mask, groups masked per element.
struct TileGroups {
  uint32_t full, bnd;
};

__device__ __forceinline__ TileGroups tile_groups(const PrefillArgs &a, int G, int64_t qb, int64_t kb) {
  int64_t dmin = 0, dmax = -1;
  TileGroups tg{0u, 0u};
  if (!tile_distance_range(a.N, BM, BN, qb, kb, &dmin, &dmax)) return tg;
  for (int g = 0; g < G; ++g) {
    const int c = classify_cutoff(dmin, dmax, a.cut[g]);
    if (c == TILE_FULL) tg.full |= 1u << g;
    if (c == TILE_BOUNDARY) tg.bnd |= 1u << g;
  }
  return tg;
}

// Smallest cutoff among the boundary groups in `bnd` that is > prev
// (prev = -1 for the first); returns false when there is none. `mask` gets
// the groups sharing that cutoff.
__device__ __forceinline__ bool next_boundary_class(const PrefillArgs &a, uint32_t bnd, int64_t prev,
                                                    int32_t *W, uint32_t *mask) {
  int64_t best = INT64_MAX;
  for (uint32_t m = bnd; m; m &= m - 1) {
    const int g = __ffs(m) - 1;
    const int64_t w = a.cut[g];
    if (w > prev && w < best) best = w;
  }
  if (best == INT64_MAX) return false;
  uint32_t mk = 0;
  for (uint32_t m = bnd; m; m &= m - 1) {
    const int g = __ffs(m) - 1;
    if (static_cast<int64_t>(a.cut[g]) == best) mk |= 1u << g;
  }
  *W = static_cast<int32_t>(best);
  *mask = mk;
  return true;
}

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    prefill_grouped_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const PrefillArgs a) {
  using L = Layout<D>;
  constexpr int G = L::G;
  constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, BN, false, false);
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, false, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::BAR_OFF);
  Barriers B;
  B.q_full = bars;
  B.k_full = bars + 1;
  B.k_empty = B.k_full + KST;
  B.v_full = B.k_empty + KST;
  B.v_empty = B.v_full + VST;
  B.s_ready = B.v_empty + VST;
  B.p_ready = B.s_ready + 2;
  B.bnd_ready = B.p_ready + 2;
  B.bnd_free = B.bnd_ready + 1;
  B.o_ready = B.bnd_free + 1;
  B.drain = B.o_ready + 1;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::MISC_OFF);
  uint32_t *tmem_base_slot = reinterpret_cast<uint32_t *>(smem + L::MISC_OFF + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int h = blockIdx.x;
  const int nqb = (a.N + BM - 1) / BM;
  const int qb = nqb - 1 - static_cast<int>(blockIdx.y);  // heaviest query tiles first
  const int b = blockIdx.z;
  const int hk = h / (a.Hq / a.Hkv);
  const long long lim = a.wait_limit;

  if (threadIdx.x == 0) {
    // An earlier CTA already gave up: skip the work, the call has failed.
    *abort_flag = *reinterpret_cast<volatile int *>(&g_status) != 0 ? 1 : 0;
    mbar_init(B.q_full, 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(&B.k_full[s], 1);
      mbar_init(&B.k_empty[s], 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(&B.v_full[s], 1);
      mbar_init(&B.v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&B.s_ready[s], 1);
      mbar_init(&B.p_ready[s], 128);
    }
    mbar_init(B.bnd_ready, 1);
    mbar_init(B.bnd_free, 128);
    mbar_init(B.o_ready, 1);
    mbar_init(B.drain, 1);
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_base_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_slot;
  const int nkb = *abort_flag ? 0 : qb + 1;  // key tiles qb, qb-1, ..., 0 (BM == BN)

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(B.q_full, G * GROUP_TILE_BYTES);
      for (int g = 0; g < G; ++g)
        tma_load_4d(smem + L::Q_OFF + g * GROUP_TILE_BYTES, &tm_q, B.q_full, 16 * g, h, qb * BM, b);
      int k_issued = 0, v_issued = 0;
      bool ok = true;
      auto load_v = [&](int t) -> bool {
        const int st = t % VST;
        if (t >= VST && !mbar_wait(&B.v_empty[st], ((t / VST) - 1) & 1, lim, abort_flag)) return false;
        const int kb = qb - t;
        mbar_arrive_expect_tx(&B.v_full[st], (D / 64) * V_CHUNK_BYTES);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(smem + L::V_OFF + st * L::V_STAGE + c * V_CHUNK_BYTES, &tm_v, &B.v_full[st], 64 * c, hk,
                      kb * BN, b);
        ++v_issued;
        return true;
      };
      for (int t = 0; ok && t < nkb; ++t) {
        const int st = t % KST;
        if (t >= KST && !mbar_wait(&B.k_empty[st], ((t / KST) - 1) & 1, lim, abort_flag)) {
          ok = false;
          break;
        }
        const int kb = qb - t;
        const TileGroups tg = tile_groups(a, G, qb, kb);
        const uint32_t need = tg.full | tg.bnd;
        mbar_arrive_expect_tx(&B.k_full[st], __popc(need) * GROUP_TILE_BYTES);
        for (uint32_t m = need; m; m &= m - 1) {
          const int g = __ffs(m) - 1;
          tma_load_4d(smem + L::K_OFF + st * L::K_STAGE + g * GROUP_TILE_BYTES, &tm_k, &B.k_full[st], 16 * g,
                      hk, kb * BN, b);
        }
        ++k_issued;
        if (t >= 1) ok = load_v(t - 1);
      }
      if (ok && nkb >= 1) ok = load_v(nkb - 1);
      // Never leave a bulk copy in flight into shared memory this CTA is
      // about to release: wait for Q and the last issued load of every stage.
      mbar_wait(B.q_full, 0, lim, nullptr);
      for (int s = 0; s < KST && s < k_issued; ++s) {
        const int last = s + ((k_issued - 1 - s) / KST) * KST;
        mbar_wait(&B.k_full[s], (last / KST) & 1, lim, nullptr);
      }
      for (int s = 0; s < VST && s < v_issued; ++s) {
        const int last = s + ((v_issued - 1 - s) / VST) * VST;
        mbar_wait(&B.v_full[s], (last / VST) & 1, lim, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(smem + L::Q_OFF);
      const uint32_t k_addr = smem_u32(smem + L::K_OFF);
      const uint32_t v_addr = smem_u32(smem + L::V_OFF);
      int bnd_issued = 0;
      bool ok = mbar_wait(B.q_full, 0, lim, abort_flag);

      auto issue_qk = [&](int t) -> bool {
        const int st = t % KST;
        if (!mbar_wait(&B.k_full[st], (t / KST) & 1, lim, abort_flag)) return false;
        tc_fence_after();
        const int kb = qb - t;
        const TileGroups tg = tile_groups(a, G, qb, kb);
        const uint32_t s_col = tmem + COL_S0 + 128u * (t & 1);
        uint32_t acc = 0;
        for (uint32_t m = tg.full; m; m &= m - 1) {
          const int g = __ffs(m) - 1;
          const uint64_t ad = smem_desc(q_addr + g * GROUP_TILE_BYTES, 16, 256, SMEM_SWIZZLE_32B);
          const uint64_t bd = smem_desc(k_addr + st * L::K_STAGE + g * GROUP_TILE_BYTES, 16, 256, SMEM_SWIZZLE_32B);
          umma_ss(s_col, ad, bd, IDESC_QK, acc);
          acc = 1;
        }
        umma_commit(&B.s_ready[t & 1]);
        int64_t prev = -1;
        int32_t W;
        uint32_t cls;
        while (next_boundary_class(a, tg.bnd, prev, &W, &cls)) {
          if (bnd_issued > 0) {
            if (!mbar_wait(B.bnd_free, (bnd_issued - 1) & 1, lim, abort_flag)) return false;
            tc_fence_after();
          }
          uint32_t bacc = 0;
          for (uint32_t m = cls; m; m &= m - 1) {
            const int g = __ffs(m) - 1;
            const uint64_t ad = smem_desc(q_addr + g * GROUP_TILE_BYTES, 16, 256, SMEM_SWIZZLE_32B);
            const uint64_t bd =
                smem_desc(k_addr + st * L::K_STAGE + g * GROUP_TILE_BYTES, 16, 256, SMEM_SWIZZLE_32B);
            umma_ss(tmem + COL_SB, ad, bd, IDESC_QK, bacc);
            bacc = 1;
          }
          umma_commit(B.bnd_ready);
          ++bnd_issued;
          prev = W;
        }
        umma_commit(&B.k_empty[st]);
        return true;
      };

      if (ok && nkb > 0) ok = issue_qk(0);
      if (ok && nkb > 1) ok = issue_qk(1);
      for (int t = 0; ok && t < nkb; ++t) {
        const int sb = t & 1;
        const int vst = t % VST;
        if (!mbar_wait(&B.p_ready[sb], (t >> 1) & 1, lim, abort_flag) ||
            !mbar_wait(&B.v_full[vst], (t / VST) & 1, lim, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t p_col = tmem + COL_S0 + 128u * sb;
        for (int kk = 0; kk < BN / 16; ++kk) {
          // V tile: 128 keys x D, dims contiguous (MN-major), 128-byte swizzle;
          // 8-key row groups 1024 B apart, 64-dim chunks 16 KB apart.
          const uint64_t bd = smem_desc(v_addr + vst * L::V_STAGE + kk * 2048, V_CHUNK_BYTES, 1024,
                                        SMEM_SWIZZLE_128B);
          umma_ts(tmem + COL_O, p_col + kk * 8, bd, IDESC_PV, (t > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&B.v_empty[vst]);
        umma_commit(B.o_ready);
        if (t + 2 < nkb) ok = issue_qk(t + 2);
      }
      // Every MMA this thread issued must finish before TMEM is released.
      umma_commit(B.drain);
      mbar_wait(B.drain, 0, lim, nullptr);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------- softmax warps
    // Every tcgen05.ld/st/wait below is .sync.aligned: the whole warp must
    // issue it together. So every wait is made warp-uniform (warp_wait), the
    // O-rescale decision is a warp vote, and only the global stores of the
    // padding rows of a ragged last tile are predicated.
    const int r = threadIdx.x;  // row of the query tile == TMEM lane
    const int64_t i = static_cast<int64_t>(qb) * BM + r;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float c2 = a.scale_log2;  // logits to base-2 exponent units
    float m_run = -INFINITY, l_run = 0.f;  // running max (base-2 units) and sum
    int bnd_used = 0;
    bool ok = true;
    for (int t = 0; t < nkb; ++t) {
      const int kb = qb - t;
      const int sb = t & 1;
      const TileGroups tg = tile_groups(a, G, qb, kb);
      if (!warp_wait(&B.s_ready[sb], (t >> 1) & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t s_addr = lane_addr + COL_S0 + 128u * sb;
      float s[BN];
      if (tg.full) {
#pragma unroll
        for (int c4 = 0; c4 < BN / 32; ++c4) {
          uint32_t u[32];
          tmem_ld32(s_addr + 32 * c4, u);
          tmem_wait_ld(u);
#pragma unroll
          for (int k = 0; k < 32; ++k) s[32 * c4 + k] = __uint_as_float(u[k]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < BN; ++c) s[c] = 0.f;
      }
      // Boundary accumulators, one distinct cutoff at a time: keep the
      // element iff its distance i - j is within the cutoff.
      int64_t prev = -1;
      int32_t W;
      uint32_t cls;
      while (next_boundary_class(a, tg.bnd, prev, &W, &cls)) {
        if (!warp_wait(B.bnd_ready, bnd_used & 1, lim, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int64_t base_dist = i - static_cast<int64_t>(kb) * BN;  // distance to key column 0
#pragma unroll
        for (int c4 = 0; c4 < BN / 32; ++c4) {
          uint32_t u[32];
          tmem_ld32(lane_addr + COL_SB + 32 * c4, u);
          tmem_wait_ld(u);
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const int c = 32 * c4 + k;
            if (base_dist - c <= static_cast<int64_t>(W)) s[c] += __uint_as_float(u[k]);
          }
        }
        tc_fence_before();
        mbar_arrive(B.bnd_free);
        ++bnd_used;
        prev = W;
      }
      if (!ok) break;
      // Causal mask: only the diagonal tile has keys after the query.
      if (kb == qb) {
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (c > r) s[c] = -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < BN; ++c) mx = fmaxf(mx, s[c]);
      const float m_tile = mx * c2;  // scale > 0, so the max commutes with it
      if (t == 0) {
        m_run = m_tile;  // the diagonal tile always holds key j = i
      } else if (__any_sync(0xffffffffu, m_tile > m_run + RESCALE_THRESHOLD)) {
        // Rescale only when some row's max grew by more than 2^8: otherwise
        // the stale max stays exact (p <= 2^8 fits bf16 P and fp32 sums).
        const float m_new = fmaxf(m_run, m_tile);
        const float alpha = fast_exp2(m_run - m_new);
        // O holds the sum through key tile t-1: wait for that PV, rescale.
        if (!warp_wait(B.o_ready, (t - 1) & 1, lim, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c4 = 0; c4 < D / 32; ++c4) {
          uint32_t u[32];
          tmem_ld32(lane_addr + COL_O + 32 * c4, u);
          tmem_wait_ld(u);
#pragma unroll
          for (int k = 0; k < 32; ++k) u[k] = __float_as_uint(__uint_as_float(u[k]) * alpha);
          tmem_st32(lane_addr + COL_O + 32 * c4, u);
        }
        tmem_wait_st();
        l_run *= alpha;
        m_run = m_new;
      }
      float rowsum = 0.f;
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t pk[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float p0 = fast_exp2(fmaf(s[64 * h2 + 2 * k], c2, -m_run));
          const float p1 = fast_exp2(fmaf(s[64 * h2 + 2 * k + 1], c2, -m_run));
          rowsum += p0 + p1;
          pk[k] = pack_bf16x2(p0, p1);
        }
        tmem_st32(s_addr + 32 * h2, pk);
      }
      l_run += rowsum;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&B.p_ready[sb]);
    }
    if (ok && nkb > 0 && warp_wait(B.o_ready, (nkb - 1) & 1, lim, abort_flag)) {
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      __nv_bfloat16 *orow = a.o + ((static_cast<int64_t>(b) * a.N + i) * a.Hq + h) * D;
#pragma unroll
      for (int c4 = 0; c4 < D / 32; ++c4) {
        uint32_t u[32];
        tmem_ld32(lane_addr + COL_O + 32 * c4, u);
        tmem_wait_ld(u);
        uint4 pk[4];
        uint32_t *pw = reinterpret_cast<uint32_t *>(pk);
#pragma unroll
        for (int k = 0; k < 16; ++k)
          pw[k] = pack_bf16x2(__uint_as_float(u[2 * k]) * inv_l, __uint_as_float(u[2 * k + 1]) * inv_l);
        if (i < a.N) {
          uint4 *dst = reinterpret_cast<uint4 *>(orow + 32 * c4);
#pragma unroll
          for (int k = 0; k < 4; ++k) dst[k] = pk[k];
        }
      }
      if (i < a.N && a.lse != nullptr)
        a.lse[(static_cast<int64_t>(b) * a.Hq + h) * a.N + i] = (m_run + log2f(l_run)) * 0.69314718055994531f;
    } else {
      // Tell the other roles to stop waiting for this warp's progress.
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

template <int D>
static cudaError_t launch_grouped(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                  const PrefillArgs &a, cudaStream_t stream) {
  const uint32_t smem = Layout<D>::ALLOC;
  cudaError_t e = cudaFuncSetAttribute(prefill_grouped_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int nqb = (a.N + BM - 1) / BM;
  dim3 grid(a.Hq, nqb, a.B);
  prefill_grouped_kernel<D><<<grid, NTHREADS, smem, stream>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

cudaError_t launch_prefill_grouped(int d_h, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                   const PrefillArgs &a, cudaStream_t stream) {
  if (d_h == 128) return launch_grouped<128>(tq, tk, tv, a, stream);
  return launch_grouped<64>(tq, tk, tv, a, stream);
}

}  // namespace wp
