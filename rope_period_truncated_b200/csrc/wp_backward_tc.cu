// WavePrune grouped-cutoff causal prefill backward on sm_100a: TMA + tcgen05 + TMEM.
//
// What it computes (WavePrune reading notes "WavePrune：RoPE 通常只需一个旋转
// 周期", §2.1 Eq. (6), §2.3 Eq. (8) and §2.3's paragraph on the backward
// kernel): with P_ij = exp(L_ij - LSE_i) from the forward's LSE and
// D_i = <dO_i, O_i>,
//   dS_ij   = P_ij (<dO_i, V_j> - D_i),
//   dQ_i[g] = scale * sum_j 1[i - j <= W_g] dS_ij K_j[g]   (16-dim group g),
// and (the key-major kernel) dV_j = sum_i P_ij dO_i, dK_j[g] likewise with Q.
// In the backward the head dimension is the output axis of the dQ and dK
// products, so the group mask goes on the gradient operand dS before the
// product: full groups take dS as it is, skipped groups nothing, a boundary
// group dS masked by its own cutoff.
//
// dq_tc_kernel: one CTA per (128-row query block, query head). It walks the
// 64-key sub-tiles from the diagonal backwards (u = 0, 1, ...; distances
// grow with u). Warp roles:
//   warp 8   TMA producer: Q and dO of the block once (16-dim boxes, 32-byte
//            swizzle); per sub-tile the K group tiles some group needs, V and
//            the sub-tile's group classes (a plan word beside the stage),
//            four stages.
//   warp 9   MMA issuer: S(u) = sum_g Q_g K_g^T (M128 N64 K16 per non-skipped
//            group) and dP(u) = dO V^T into the S/dP buffer of TMEM, then,
//            once the row warps have written dS(u) (bf16) into one of the two
//            operand buffers, dQ[g0:g1] += dS K[g0:g1] for each run of
//            consecutive full groups as M128 N16*(g1-g0) K16 products with dS
//            read from TMEM and K read MN-major from the same swizzled group
//            tiles.
//   warps 0-7 two threads per query row: warp w reads TMEM lanes 32 (w % 4)..
//            and the sub-tile's columns 32 (w / 4) .. +31, and forms P and
//            dS = P (dP - D) there in packed f32x2 arithmetic (no row
//            reduction is needed: P comes from the forward's LSE). S and dP
//            have one TMEM buffer: the row warps release it as soon as they
//            have loaded it, so S(u + 1) runs on the tensor cores while they
//            compute u, and they write dS as bf16 into one of two operand
//            buffers that the dQ products read. The epilogue scales dQ and
//            writes it as bf16.
// Boundary groups (cutoff inside the sub-tile's distance range), as in the
// forward kernel: their S products go first, one cutoff class at a time in
// ascending order, and the row warps mask S in place after each (nested
// windows: the exact per-group mask). For dQ the classes go in descending
// order: before each class's products the row warps overwrite dS in TMEM
// with dS masked by that class's cutoff. Both are round trips between the
// MMA warp and the row warps, so the MMA warp issues S(v) of a sub-tile with
// boundary classes only after it has issued dQ(v - 1): the row warps finish
// sub-tile v - 1 before they mask S(v), and the MMA warp never waits on them
// for a later sub-tile.
// (Without boundary classes, S(v) goes out as soon as the row warps have
// loaded S(v - 1).)
//
// dkdv_tc_kernel: one CTA per (128-row key block, KV head), the same roles
// with keys as rows: K and V of the block once; per 64-query sub-tile (the
// KV head's query heads one after another, each from the diagonal outwards)
// Q, dO and their LSE and D. S^T = K Q^T and dP^T = V dO^T on the tensor
// cores, P^T and dS^T per key row, then dV += P^T dO (N = d) and
// dK[g0:g1] += dS^T Q[g0:g1] per run of full groups; the query heads of the
// KV head add into the same TMEM accumulators, so nothing is reduced across
// CTAs. Boundary classes as above, with the window on the query columns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "wp_backward.h"
#include "wp_device.cuh"
#include "wp_prefill_common.cuh"
#include "wp_tile.h"

namespace wp {

namespace {

constexpr int TBQ = 128;  // rows of a CTA's block
constexpr int TBS = 64;   // columns of a sub-tile
constexpr int TNST = 4;   // stages of the streamed operands
constexpr int CSPLIT = 2;               // row warps per TMEM lane quarter: the sub-tile's columns split
constexpr int COLS = TBS / CSPLIT;      // columns of one row warp
constexpr int NROWW = 4 * CSPLIT;       // row warps
constexpr int TC_THREADS = 32 * (NROWW + 2);  // + TMA producer, MMA issuer
constexpr int T_PROD = NROWW, T_MMA = NROWW + 1;
static_assert(COLS == 16 || COLS == 32, "row warps take 16 or 32 columns");
constexpr uint32_t TILE128 = 128 * 32;  // a 16-dim group tile of 128 rows
constexpr uint32_t TILE64 = 64 * 32;    // a 16-dim group tile of 64 rows
constexpr float TLOG2E = 1.4426950408889634f;

// A sub-tile's group classes: bits 0-7 full groups, 8-15 boundary groups,
// bit 16 set when the sub-tile holds causal pairs at all.
__device__ __forceinline__ uint32_t plan_word(const int32_t *cut, int G, bool any, int64_t dmin, int64_t dmax) {
  uint32_t full = 0, bnd = 0;
  if (any) {
    for (int g = 0; g < G; ++g) {
      const int c = classify_cutoff(dmin, dmax, cut[g]);
      if (c == TILE_FULL) full |= 1u << g;
      if (c == TILE_BOUNDARY) bnd |= 1u << g;
    }
  }
  return full | (bnd << 8) | (any ? 1u << 16 : 0u);
}
__device__ __forceinline__ uint32_t pw_full(uint32_t w) { return w & 0xffu; }
__device__ __forceinline__ uint32_t pw_bnd(uint32_t w) { return (w >> 8) & 0xffu; }
__device__ __forceinline__ bool pw_any(uint32_t w) { return (w >> 16) & 1u; }

// Largest cutoff among the boundary groups in `bnd` that is < prev (prev =
// INT64_MAX for the first); false when none. `mask` gets the groups of it.
__device__ __forceinline__ bool prev_boundary_class(const int32_t *cut, uint32_t bnd, int64_t prev, int32_t *W,
                                                    uint32_t *mask) {
  int64_t best = -1;
  for (uint32_t m = bnd; m; m &= m - 1) {
    const int64_t w = cut[__ffs(m) - 1];
    if (w < prev && w > best) best = w;
  }
  if (best < 0) return false;
  uint32_t mk = 0;
  for (uint32_t m = bnd; m; m &= m - 1) {
    const int g = __ffs(m) - 1;
    if (static_cast<int64_t>(cut[g]) == best) mk |= 1u << g;
  }
  *W = static_cast<int32_t>(best);
  *mask = mk;
  return true;
}

// 4-byte asynchronous copy global -> shared; src_bytes 0 writes zero.
__device__ __forceinline__ void cp_async4(void *dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
// The barrier's current phase also waits for this thread's earlier cp.async
// copies (its pending count rises now and falls when they land).
__device__ __forceinline__ void cp_async_arrive(uint64_t *bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15])
               :
               : "memory");
}
[[maybe_unused]] __device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

// COLS TMEM columns of this warp's lanes into r (and waited for).
template <int NC>
__device__ __forceinline__ void ld_cols(uint32_t taddr, uint32_t (&r)[NC]) {
  if constexpr (NC == 32) {
    tmem_ld32(taddr, r);
    tmem_wait_ld(r);
  } else {
    tmem_ld16(taddr, r);
    tmem_wait_ld16(r);
  }
}
// COLS columns at each of two addresses, one wait for both.
template <int NC>
__device__ __forceinline__ void ld_cols2(uint32_t a0, uint32_t (&r0)[NC], uint32_t a1, uint32_t (&r1)[NC]) {
  if constexpr (NC == 32) {
    tmem_ld32(a0, r0);
    tmem_ld32(a1, r1);
    tmem_wait_ld(r0);
    tmem_wait_ld(r1);
  } else {
    tmem_ld16(a0, r0);
    tmem_ld16(a1, r1);
    tmem_wait_ld16(r0);
    tmem_wait_ld16(r1);
  }
}
template <int NC>
__device__ __forceinline__ void st_cols(uint32_t taddr, const uint32_t (&r)[NC]) {
  if constexpr (NC == 32)
    tmem_st32(taddr, r);
  else
    tmem_st16(taddr, r);
}

// COLS fp32 values as bf16 pairs into COLS / 2 TMEM columns; columns outside
// [lo, hi] (0-based within the COLS) written as 0.
template <int NC>
__device__ __forceinline__ void store_bf16_cols(uint32_t taddr, const float (&x)[NC], int lo, int hi) {
  uint32_t pk[NC / 2];
#pragma unroll
  for (int k = 0; k < NC / 2; ++k)
    pk[k] = pack_bf16x2(2 * k < lo || 2 * k > hi ? 0.f : x[2 * k], 2 * k + 1 < lo || 2 * k + 1 > hi ? 0.f : x[2 * k + 1]);
  if constexpr (NC == 32)
    tmem_st16(taddr, pk);
  else
    tmem_st8(taddr, pk);
}

// Zero n16 x 16 TMEM columns of this warp's lanes.
__device__ __forceinline__ void tmem_zero16(uint32_t taddr, int n16) {
  uint32_t z[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) z[k] = 0u;
  for (int c = 0; c < n16; ++c) tmem_st16(taddr + 16 * c, z);
  tmem_wait_st();
}

// Scale 16 fp32 TMEM columns, write them to global memory as bf16 (16-byte stores).
__device__ __forceinline__ void store_row16(uint32_t taddr, float scale, __nv_bfloat16 *dst, bool ok) {
  uint32_t u16[16];
  tmem_ld16(taddr, u16);
  tmem_wait_ld16(u16);
  uint4 pk4[2];
  uint32_t *pw = reinterpret_cast<uint32_t *>(pk4);
#pragma unroll
  for (int k = 0; k < 8; ++k)
    pw[k] = pack_bf16x2(__uint_as_float(u16[2 * k]) * scale, __uint_as_float(u16[2 * k + 1]) * scale);
  if (ok) {
    reinterpret_cast<uint4 *>(dst)[0] = pk4[0];
    reinterpret_cast<uint4 *>(dst)[1] = pk4[1];
  }
}

__device__ __forceinline__ void store_nan(__nv_bfloat16 *dst, int n) {
  const uint4 nan4 = make_uint4(0x7FC07FC0u, 0x7FC07FC0u, 0x7FC07FC0u, 0x7FC07FC0u);
  for (int k = 0; k < n / 8; ++k) reinterpret_cast<uint4 *>(dst)[k] = nan4;
}

// ============================================================ dQ kernel

// TMEM columns of the dQ kernel
constexpr uint32_t DQ_S = 0;     // S (fp32, 64 columns)
constexpr uint32_t DQ_DP = 64;   // dP
constexpr uint32_t DQ_OB = 128;  // dS as bf16, operand buffer b at 128 + 32 b
constexpr uint32_t DQ_ACC = 256;

template <int D>
struct DqTL {
  static constexpr int G = D / 16;
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t DO_OFF = Q_OFF + G * TILE128;
  static constexpr uint32_t K_OFF = DO_OFF + G * TILE128;
  static constexpr uint32_t STAGE = G * TILE64;
  static constexpr uint32_t V_OFF = K_OFF + TNST * STAGE;
  static constexpr uint32_t BAR_OFF = V_OFF + TNST * STAGE;
  // qd_full, kv_full[TNST], kv_empty[TNST], s_ready, s_free, ds_ready[2],
  // ob_free[2], bnd_ready, bnd_done, dsm_req, dsm_done, dq_final, drain
  static constexpr uint32_t NUM_BARS = 1 + 2 * TNST + 12;
  static constexpr uint32_t MISC_OFF = BAR_OFF + NUM_BARS * 8;
  static constexpr uint32_t CUT_OFF = MISC_OFF + 16;  // the head's group cutoffs, 8 int32
  static constexpr uint32_t PLAN_OFF = CUT_OFF + 32;  // plan word per stage
  static constexpr uint32_t BYTES = PLAN_OFF + 4 * TNST + 1024;
};

template <int D>
__global__ void __launch_bounds__(TC_THREADS, 1)
    dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                 const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 const __grid_constant__ BackwardArgs a) {
  using L = DqTL<D>;
  constexpr int G = L::G;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(128, TBS, false, false);
  constexpr uint32_t GD128 = TILE128 >> 4, GD64 = TILE64 >> 4;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::BAR_OFF);
  uint64_t *qd_full = bars;
  uint64_t *kv_full = bars + 1;
  uint64_t *kv_empty = kv_full + TNST;
  uint64_t *s_ready = kv_empty + TNST, *s_free = s_ready + 1;
  uint64_t *ds_ready = s_free + 1;   // [2 operand buffers]
  uint64_t *ob_free = ds_ready + 2;  // [2 operand buffers]
  uint64_t *bnd_ready = ob_free + 2, *bnd_done = bnd_ready + 1, *dsm_req = bnd_done + 1, *dsm_done = dsm_req + 1;
  uint64_t *dq_final = dsm_done + 1, *drain = dq_final + 1;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::MISC_OFF);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::MISC_OFF + 4);
  int32_t *cut = reinterpret_cast<int32_t *>(smem + L::CUT_OFF);
  volatile uint32_t *plans = reinterpret_cast<volatile uint32_t *>(smem + L::PLAN_OFF);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.y, b = blockIdx.z;
  const int hk = h / (a.Hq / a.Hkv);
  const int nqb = (a.N + TBQ - 1) / TBQ;
  const int qb = nqb - 1 - static_cast<int>(blockIdx.x);  // heaviest blocks first
  const int64_t N = a.N;
  const long long lim = a.wait_limit;

  if (threadIdx.x == 0) {
    *abort_flag = *reinterpret_cast<volatile int *>(&g_status) != 0 ? 1 : 0;
    mbar_init(qd_full, 1);
    for (int s = 0; s < TNST; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(s_ready, 1);
    mbar_init(s_free, NROWW);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ds_ready[s], NROWW);
      mbar_init(&ob_free[s], 1);
    }
    mbar_init(bnd_ready, 1);
    mbar_init(bnd_done, NROWW);
    mbar_init(dsm_req, 1);
    mbar_init(dsm_done, NROWW);
    mbar_init(dq_final, 1);
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (threadIdx.x < 8) cut[threadIdx.x] = threadIdx.x < G ? a.cut[(a.cut_rows == 1 ? 0 : h) * G + threadIdx.x] : 0;
  if (warp == T_MMA) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nsub = *abort_flag ? 0 : 2 * (qb + 1);  // key sub-tile 2qb + 1 - u

  if (warp == T_PROD) {
    // ------------------------------------------------------------ producer
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(qd_full, 2 * G * TILE128);
      for (int g = 0; g < G; ++g) {
        tma_load_4d(smem + L::Q_OFF + g * TILE128, &tm_q, qd_full, 16 * g, h, qb * TBQ, b);
        tma_load_4d(smem + L::DO_OFF + g * TILE128, &tm_do, qd_full, 16 * g, h, qb * TBQ, b);
      }
    }
    __syncwarp();
    int issued = 0;
    for (int u = 0; u < nsub; ++u) {
      const int st = u % TNST;
      if (u >= TNST && !warp_wait_idle<32>(&kv_empty[st], ((u / TNST) - 1) & 1, lim, abort_flag)) break;
      int64_t dmin = 0, dmax = -1;
      const bool any = tile_distance_range(N, TBQ, TBS, qb, 2 * qb + 1 - u, &dmin, &dmax);
      const uint32_t w = plan_word(cut, G, any, dmin, dmax);
      if (lane == 0) plans[st] = w;
      __syncwarp();
      // a sub-tile without causal pairs (past the end of a ragged last block)
      // loads nothing: its dS is 0 whatever the buffers hold
      const uint32_t need = pw_full(w) | pw_bnd(w);
      const int nv = any ? G : 0;
      const int krow = (2 * qb + 1 - u) * TBS;
      if (leader) {
        mbar_arrive_expect_tx(&kv_full[st], (__popc(need) + nv) * TILE64);
        for (uint32_t m = need; m; m &= m - 1) {
          const int g = __ffs(m) - 1;
          tma_load_4d(smem + L::K_OFF + st * L::STAGE + g * TILE64, &tm_k, &kv_full[st], 16 * g, hk, krow, b);
        }
        for (int g = 0; g < nv; ++g)
          tma_load_4d(smem + L::V_OFF + st * L::STAGE + g * TILE64, &tm_v, &kv_full[st], 16 * g, hk, krow, b);
      }
      __syncwarp();
      ++issued;
    }
    warp_wait_idle(qd_full, 0, lim, nullptr);
    for (int s = 0; s < TNST && s < issued; ++s) {
      const int last = s + ((issued - 1 - s) / TNST) * TNST;
      warp_wait_idle(&kv_full[s], (last / TNST) & 1, lim, nullptr);
    }
  } else if (warp == T_MMA) {
    // -------------------------------------------------------- MMA issuer
    const bool leader = elect_one();
    const uint64_t q_desc = smem_desc(smem_u32(smem + L::Q_OFF), 16, 256, SMEM_SWIZZLE_32B);
    const uint64_t do_desc = smem_desc(smem_u32(smem + L::DO_OFF), 16, 256, SMEM_SWIZZLE_32B);
    const uint64_t k_desc = smem_desc(smem_u32(smem + L::K_OFF), 16, 256, SMEM_SWIZZLE_32B);
    const uint64_t v_desc = smem_desc(smem_u32(smem + L::V_OFF), 16, 256, SMEM_SWIZZLE_32B);
    // K as the B operand of dQ += dS K: keys along K (8-row groups 256 B
    // apart), dims along N (16-dim group tiles TILE64 apart)
    const uint64_t kmn_desc = smem_desc(smem_u32(smem + L::K_OFF), TILE64, 256, SMEM_SWIZZLE_32B);
    bool ok = warp_wait(qd_full, 0, lim, abort_flag);
    int bnd_cnt = 0, dsm_cnt = 0;

    auto plan = [&](int u, uint32_t &w) -> bool {
      if (!warp_wait(&kv_full[u % TNST], (u / TNST) & 1, lim, abort_flag)) return false;
      w = plans[u % TNST];
      return true;
    };
    // S(u) and dP(u) into the S buffer (its stage loaded, S(u - 1) loaded by the row warps)
    auto issue_sdp = [&](int u, uint32_t w) -> bool {
      const int st = u % TNST;
      tc_fence_after();
      const uint32_t s_col = tmem + DQ_S;
      const uint64_t kst = k_desc + ((st * L::STAGE) >> 4);
      uint32_t acc = 0;
      if (pw_bnd(w)) {
        int64_t prev = -1;
        int32_t W;
        uint32_t cls;
        while (next_boundary_class(cut, pw_bnd(w), prev, &W, &cls)) {
          if (leader) {
            for (int g = 0; g < G; ++g)
              if ((cls >> g) & 1u) {
                umma_ss(s_col, q_desc + g * GD128, kst + g * GD64, IDESC_S, acc);
                acc = 1;
              }
            umma_commit(bnd_ready);
          }
          acc = 1;
          __syncwarp();
          if (!warp_wait(bnd_done, bnd_cnt & 1, lim, abort_flag)) return false;
          tc_fence_after();
          ++bnd_cnt;
          prev = W;
        }
      }
      if (leader) {
        const uint32_t full = pw_full(w);
#pragma unroll
        for (int g = 0; g < G; ++g)
          if ((full >> g) & 1u) {
            umma_ss(s_col, q_desc + g * GD128, kst + g * GD64, IDESC_S, acc);
            acc = 1;
          }
        const uint64_t vst = v_desc + ((st * L::STAGE) >> 4);
        if (pw_any(w)) {
#pragma unroll
          for (int g = 0; g < G; ++g)
            umma_ss(tmem + DQ_DP, do_desc + g * GD128, vst + g * GD64, IDESC_S, g > 0 ? 1u : 0u);
        }
        umma_commit(s_ready);
      }
      __syncwarp();
      return true;
    };
    // dQ[groups] += dS(u) K[groups], one product set per run of consecutive groups
    auto issue_dq_groups = [&](int u, uint32_t groups) {
      const int st = u % TNST;
      const uint64_t kst = kmn_desc + ((st * L::STAGE) >> 4);
      const uint32_t ob = tmem + DQ_OB + 32 * (u & 1);
      while (groups) {
        const int g0 = __ffs(groups) - 1;
        int g1 = g0;
        while (g1 < G && ((groups >> g1) & 1u)) ++g1;
        groups &= ~(((1u << g1) - 1u) & ~((1u << g0) - 1u));
        const uint32_t idesc = idesc_bf16_f32(128, 16 * (g1 - g0), false, true);
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < TBS / 16; ++kk)
            umma_ts(tmem + DQ_ACC + 16 * g0, ob + 8 * kk, kst + g0 * GD64 + ((kk * 16 * 32) >> 4), idesc, 1u);
        }
        __syncwarp();
      }
    };
    // dQ(u): full groups on dS as it is, then the boundary classes in
    // descending cutoff order, each after the row warps masked dS for it
    auto issue_dq = [&](int u) -> bool {
      const uint32_t w = plans[u % TNST];
      issue_dq_groups(u, pw_full(w));
      int64_t prev = INT64_MAX;
      int32_t W;
      uint32_t cls;
      while (prev_boundary_class(cut, pw_bnd(w), prev, &W, &cls)) {
        if (leader) umma_commit(dsm_req);
        __syncwarp();
        if (!warp_wait(dsm_done, dsm_cnt & 1, lim, abort_flag)) return false;
        tc_fence_after();
        ++dsm_cnt;
        issue_dq_groups(u, cls);
        prev = W;
      }
      if (leader) {
        umma_commit(&kv_empty[u % TNST]);
        umma_commit(&ob_free[u & 1]);
      }
      __syncwarp();
      return true;
    };
    // S(v + 1) once the row warps have loaded S(v)
    auto next_sdp = [&](int v) -> bool {
      uint32_t w;
      if (!warp_wait(s_free, v & 1, lim, abort_flag) || !plan(v + 1, w)) return false;
      return issue_sdp(v + 1, w);
    };

    if (ok && nsub > 0) {
      uint32_t w;
      ok = plan(0, w) && issue_sdp(0, w);
    }
    for (int u = 0; ok && u < nsub; ++u) {
      // S(u + 1) overlaps the row warps' work on u, unless it has boundary
      // classes: then its handshakes follow dQ(u) and the row warps' masking for u
      bool early = false;
      if (u + 1 < nsub) {
        uint32_t w1;
        if (!plan(u + 1, w1)) {
          ok = false;
          break;
        }
        if (pw_bnd(w1) == 0u) {
          early = true;
          if (!(ok = next_sdp(u))) break;
        }
      }
      if (!warp_wait(&ds_ready[u & 1], (u >> 1) & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      ok = issue_dq(u);
      if (ok && u + 1 < nsub && !early) ok = next_sdp(u);
    }
    if (leader) {
      umma_commit(dq_final);
      umma_commit(drain);
    }
    __syncwarp();
    warp_wait(drain, 0, lim, nullptr);
  } else if (warp < NROWW) {
    // ---------------------------------------------------------- row warps
    const int q4 = warp & 3, cq = warp >> 2, cb = COLS * cq;  // lane quarter, first column
    const int r = q4 * 32 + lane;
    const int64_t i = static_cast<int64_t>(qb) * TBQ + r;
    const bool row_ok = i < N;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const uint32_t s_addr = lane_addr + DQ_S + cb, dp_addr = lane_addr + DQ_DP + cb;
    const int64_t lrow = (static_cast<int64_t>(b) * a.Hq + h) * a.N + (row_ok ? i : 0);
    const float lse2 = row_ok ? a.lse[lrow] * TLOG2E : 0.f;
    const float di = row_ok ? a.delta[lrow] : 0.f;
    const uint64_t c2x2 = pack_f2(a.scale_log2, a.scale_log2), nl2 = pack_f2(-lse2, -lse2), nd2 = pack_f2(-di, -di);
    constexpr int DPW = D / CSPLIT;  // accumulator columns of this warp in the epilogue
    tmem_zero16(lane_addr + DQ_ACC + cq * DPW, DPW / 16);  // every dQ product accumulates
    int bnd_cnt = 0, dsm_cnt = 0;
    bool ok = true;
    for (int u = 0; ok && u < nsub; ++u) {
      const int st = u % TNST;
      const int64_t k0 = static_cast<int64_t>(2 * qb + 1 - u) * TBS + cb;  // first key of my columns
      const uint32_t ob_addr = lane_addr + DQ_OB + 32 * (u & 1) + (COLS / 2) * cq;
      if (!warp_wait(&kv_full[st], (u / TNST) & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      const uint32_t w = plans[st];
      if (pw_bnd(w)) {
        // S masked in place after each boundary class: keep key c iff i - (k0 + c) <= W
        int64_t prev = -1;
        int32_t W;
        uint32_t cls;
        while (next_boundary_class(cut, pw_bnd(w), prev, &W, &cls)) {
          ok = warp_wait(bnd_ready, bnd_cnt & 1, lim, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const int64_t cm = i - k0 - W;
          const int cmin = cm < 0 ? 0 : (cm > COLS ? COLS : static_cast<int>(cm));
          uint32_t su[COLS];
          ld_cols(s_addr, su);
#pragma unroll
          for (int c = 0; c < COLS; ++c)
            if (c < cmin) su[c] = 0u;
          st_cols(s_addr, su);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bnd_done);
          ++bnd_cnt;
          prev = W;
        }
        if (!ok) break;
      }
      // a sleeping poll: a spinning row warp would take issue slots from the
      // MMA warp that shares its scheduler, which is what S(u) waits for
      if (!warp_wait_idle<32>(s_ready, u & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // No S product for this sub-tile: its S is 0. Store the zeros into this
      // warp's S columns (no MMA reads them) so that every sub-tile takes the
      // same loads; zeroing the registers on that path instead gives them two
      // definitions, and the merge costs register moves on every sub-tile.
      if (!(pw_full(w) | pw_bnd(w))) tmem_zero16(s_addr, COLS / 16);
      uint32_t su[COLS], dp[COLS];
      ld_cols2(s_addr, su, dp_addr, dp);
      // S and dP are in registers: the buffer is free for S(u + 1)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);
      // P = exp2(S c2 - LSE log2 e) and dS = P (dP - D) on the causal pairs of a valid row
      const int64_t jm = i - k0;  // my last causal column
      const int jmax = !row_ok ? -1 : (jm > COLS - 1 ? COLS - 1 : (jm < -1 ? -1 : static_cast<int>(jm)));
      float ds[COLS];
#pragma unroll
      for (int k = 0; k < COLS / 2; ++k) {
        const uint64_t x2 = ffma2(pack_f2(__uint_as_float(su[2 * k]), __uint_as_float(su[2 * k + 1])), c2x2, nl2);
        float x0, x1;
        unpack_f2(x2, x0, x1);
        const uint64_t g2 = fadd2(pack_f2(__uint_as_float(dp[2 * k]), __uint_as_float(dp[2 * k + 1])), nd2);
        float d0, d1;
        unpack_f2(fmul2(pack_f2(fast_exp2(x0), fast_exp2(x1)), g2), d0, d1);
        ds[2 * k] = d0;
        ds[2 * k + 1] = d1;
      }
      // operand buffer u & 1 is free once dQ(u - 2) has read it
      if (u >= 2 && !warp_wait(&ob_free[u & 1], ((u >> 1) - 1) & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      store_bf16_cols(ob_addr, ds, 0, jmax);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ds_ready[u & 1]);
      // boundary classes of dQ, descending cutoffs: dS masked for each
      int64_t prev = INT64_MAX;
      int32_t W;
      uint32_t cls;
      while (prev_boundary_class(cut, pw_bnd(w), prev, &W, &cls)) {
        ok = warp_wait(dsm_req, dsm_cnt & 1, lim, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const int64_t cm = i - k0 - W;
        store_bf16_cols(ob_addr, ds, cm < 0 ? 0 : (cm > COLS ? COLS : static_cast<int>(cm)), jmax);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dsm_done);
        ++dsm_cnt;
        prev = W;
      }
    }
    __nv_bfloat16 *dqrow = a.dq + ((static_cast<int64_t>(b) * a.N + i) * a.Hq + h) * D + cq * DPW;
    if (ok && nsub > 0 && warp_wait(dq_final, 0, lim, abort_flag)) {
      tc_fence_after();
      for (int c = 0; c < DPW / 16; ++c)
        store_row16(lane_addr + DQ_ACC + cq * DPW + 16 * c, a.scale, dqrow + 16 * c, row_ok);
    } else {
      *abort_flag = 1;
      if (row_ok) store_nan(dqrow, DPW);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == T_MMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ========================================================= dK/dV kernel

// TMEM columns of the dK/dV kernel
constexpr uint32_t KV_S = 0;     // S^T (fp32, 64 columns)
constexpr uint32_t KV_DP = 64;   // dP^T
constexpr uint32_t KV_OB = 128;  // operand buffer b at 128 + 64 b: P^T (bf16, 32 columns), then dS^T
constexpr uint32_t KV_DK = 256;

template <int D>
struct KvTL {
  static constexpr int G = D / 16;
  static constexpr uint32_t DV_COL = KV_DK + D;
  static constexpr uint32_t K_OFF = 0;
  static constexpr uint32_t V_OFF = K_OFF + G * TILE128;
  static constexpr uint32_t Q_OFF = V_OFF + G * TILE128;
  static constexpr uint32_t STAGE = G * TILE64;
  static constexpr uint32_t DO_OFF = Q_OFF + TNST * STAGE;
  static constexpr uint32_t LD_OFF = DO_OFF + TNST * STAGE;  // per stage: LSE and D of the 64 queries
  static constexpr uint32_t BAR_OFF = LD_OFF + TNST * 512;
  // kv_full, qd_full[TNST], qd_empty[TNST], s_ready, s_free, ds_ready[2],
  // ob_free[2], bnd_ready, bnd_done, dsm_req, dsm_done, kv_final, drain
  static constexpr uint32_t NUM_BARS = 1 + 2 * TNST + 12;
  static constexpr uint32_t MISC_OFF = BAR_OFF + NUM_BARS * 8;
  static constexpr uint32_t PLAN_OFF = MISC_OFF + 16;       // plan word and head of each stage
  static constexpr uint32_t CUT_OFF = PLAN_OFF + 8 * TNST;  // cutoff rows of the KV head's query heads, [rep][8]
  static constexpr uint32_t BYTES = CUT_OFF + 64 * 8 * 4 + 1024;
};

template <int D>
__global__ void __launch_bounds__(TC_THREADS, 1)
    dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ BackwardArgs a) {
  using L = KvTL<D>;
  constexpr int G = L::G;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(128, TBS, false, false);
  constexpr uint32_t GD128 = TILE128 >> 4, GD64 = TILE64 >> 4;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::BAR_OFF);
  uint64_t *kv_full = bars;
  uint64_t *qd_full = bars + 1;
  uint64_t *qd_empty = qd_full + TNST;
  uint64_t *s_ready = qd_empty + TNST, *s_free = s_ready + 1;
  uint64_t *ds_ready = s_free + 1;   // [2 operand buffers]
  uint64_t *ob_free = ds_ready + 2;  // [2 operand buffers]
  uint64_t *bnd_ready = ob_free + 2, *bnd_done = bnd_ready + 1, *dsm_req = bnd_done + 1, *dsm_done = dsm_req + 1;
  uint64_t *kv_final = dsm_done + 1, *drain = kv_final + 1;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::MISC_OFF);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::MISC_OFF + 4);
  volatile uint32_t *plans = reinterpret_cast<volatile uint32_t *>(smem + L::PLAN_OFF);  // [stage]
  int32_t *cuts = reinterpret_cast<int32_t *>(smem + L::CUT_OFF);                        // [rep][8]

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int kb = static_cast<int>(blockIdx.x);  // key blocks near the start see the most queries: first
  const int hk = blockIdx.y, b = blockIdx.z;
  const int rep = a.Hq / a.Hkv;
  const int64_t N = a.N;
  const int nq64 = (a.N + TBS - 1) / TBS;
  const int per_head = nq64 - 2 * kb;  // query sub-tiles 2kb .. nq64-1 of each head
  const long long lim = a.wait_limit;

  if (threadIdx.x == 0) {
    *abort_flag = *reinterpret_cast<volatile int *>(&g_status) != 0 ? 1 : 0;
    mbar_init(kv_full, 1);
    for (int s = 0; s < TNST; ++s) {
      mbar_init(&qd_full[s], 1);
      mbar_init(&qd_empty[s], 1);
    }
    mbar_init(s_ready, 1);
    mbar_init(s_free, NROWW);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ds_ready[s], NROWW);
      mbar_init(&ob_free[s], 1);
    }
    mbar_init(bnd_ready, 1);
    mbar_init(bnd_done, NROWW);
    mbar_init(dsm_req, 1);
    mbar_init(dsm_done, NROWW);
    mbar_init(kv_final, 1);
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  for (int x = threadIdx.x; x < rep * 8; x += TC_THREADS) {
    const int hr = x / 8, g = x % 8;
    cuts[x] = g < G ? a.cut[(a.cut_rows == 1 ? 0 : hk * rep + hr) * G + g] : 0;
  }
  if (warp == T_MMA) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nsub = *abort_flag ? 0 : rep * per_head;
  // sub-tile u: query head hk * rep + u / per_head, query rows 64 * (2kb + u % per_head) ..
  auto q0_of = [&](int u) { return static_cast<int64_t>(2 * kb + u % per_head) * TBS; };

  if (warp == T_PROD) {
    // ------------------------------------------------------------ producer
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(kv_full, 2 * G * TILE128);
      for (int g = 0; g < G; ++g) {
        tma_load_4d(smem + L::K_OFF + g * TILE128, &tm_k, kv_full, 16 * g, hk, kb * TBQ, b);
        tma_load_4d(smem + L::V_OFF + g * TILE128, &tm_v, kv_full, 16 * g, hk, kb * TBQ, b);
      }
    }
    __syncwarp();
    int issued = 0;
    for (int u = 0; u < nsub; ++u) {
      const int st = u % TNST;
      if (u >= TNST && !warp_wait_idle<32>(&qd_empty[st], ((u / TNST) - 1) & 1, lim, abort_flag)) break;
      const int hr = u / per_head;
      const int h = hk * rep + hr;
      const int64_t q0 = q0_of(u);
      int64_t dmin = 0, dmax = -1;
      const bool any = tile_distance_range(N, TBS, TBQ, 2 * kb + u % per_head, kb, &dmin, &dmax);
      const uint32_t w = plan_word(cuts + 8 * hr, G, any, dmin, dmax);
      // The bulk copies go out first, then the sub-tile's LSE and D as
      // asynchronous 4-byte copies (zero past N) tracked by the same barrier,
      // and the plan; the arrival that carries the expected bytes comes last
      // (the copies' completions may precede it: the phase waits for all).
      const uint32_t need = pw_full(w) | pw_bnd(w);
      if (leader) {
        for (uint32_t m = need; m; m &= m - 1) {
          const int g = __ffs(m) - 1;
          tma_load_4d(smem + L::Q_OFF + st * L::STAGE + g * TILE64, &tm_q, &qd_full[st], 16 * g, h,
                      static_cast<int>(q0), b);
        }
        for (int g = 0; g < G; ++g)
          tma_load_4d(smem + L::DO_OFF + st * L::STAGE + g * TILE64, &tm_do, &qd_full[st], 16 * g, h,
                      static_cast<int>(q0), b);
      }
      float *ld = reinterpret_cast<float *>(smem + L::LD_OFF + st * 512);
      const int64_t lrow = (static_cast<int64_t>(b) * a.Hq + h) * a.N;
      for (int c = lane; c < TBS; c += 32) {
        const bool in = q0 + c < N;
        const int64_t e = lrow + (in ? q0 + c : 0);
        cp_async4(ld + c, a.lse + e, in ? 4u : 0u);
        cp_async4(ld + TBS + c, a.delta + e, in ? 4u : 0u);
      }
      cp_async_arrive(&qd_full[st]);
      if (lane == 0) {
        plans[2 * st] = w;
        plans[2 * st + 1] = static_cast<uint32_t>(hr);
      }
      __syncwarp();
      if (leader) mbar_arrive_expect_tx(&qd_full[st], (__popc(need) + G) * TILE64);
      __syncwarp();
      ++issued;
    }
    warp_wait_idle(kv_full, 0, lim, nullptr);
    for (int s = 0; s < TNST && s < issued; ++s) {
      const int last = s + ((issued - 1 - s) / TNST) * TNST;
      warp_wait_idle(&qd_full[s], (last / TNST) & 1, lim, nullptr);
    }
  } else if (warp == T_MMA) {
    // -------------------------------------------------------- MMA issuer
    const bool leader = elect_one();
    const uint64_t k_desc = smem_desc(smem_u32(smem + L::K_OFF), 16, 256, SMEM_SWIZZLE_32B);
    const uint64_t v_desc = smem_desc(smem_u32(smem + L::V_OFF), 16, 256, SMEM_SWIZZLE_32B);
    const uint64_t q_desc = smem_desc(smem_u32(smem + L::Q_OFF), 16, 256, SMEM_SWIZZLE_32B);
    const uint64_t do_desc = smem_desc(smem_u32(smem + L::DO_OFF), 16, 256, SMEM_SWIZZLE_32B);
    // Q and dO as the B operands of the dK and dV products: queries along K,
    // dims along N (16-dim group tiles TILE64 apart)
    const uint64_t qmn_desc = smem_desc(smem_u32(smem + L::Q_OFF), TILE64, 256, SMEM_SWIZZLE_32B);
    const uint64_t domn_desc = smem_desc(smem_u32(smem + L::DO_OFF), TILE64, 256, SMEM_SWIZZLE_32B);
    bool ok = warp_wait(kv_full, 0, lim, abort_flag);
    int bnd_cnt = 0, dsm_cnt = 0;

    auto plan = [&](int u, uint32_t &w) -> bool {
      if (!warp_wait(&qd_full[u % TNST], (u / TNST) & 1, lim, abort_flag)) return false;
      w = plans[2 * (u % TNST)];
      return true;
    };
    // S^T(u) and dP^T(u) into the S buffer
    auto issue_sdp = [&](int u, uint32_t w) -> bool {
      const int st = u % TNST;
      tc_fence_after();
      const int32_t *cut = cuts + 8 * static_cast<int>(plans[2 * st + 1]);
      const uint32_t s_col = tmem + KV_S;
      const uint64_t qst = q_desc + ((st * L::STAGE) >> 4);
      uint32_t acc = 0;
      if (pw_bnd(w)) {
        int64_t prev = -1;
        int32_t W;
        uint32_t cls;
        while (next_boundary_class(cut, pw_bnd(w), prev, &W, &cls)) {
          if (leader) {
            for (int g = 0; g < G; ++g)
              if ((cls >> g) & 1u) {
                umma_ss(s_col, k_desc + g * GD128, qst + g * GD64, IDESC_S, acc);
                acc = 1;
              }
            umma_commit(bnd_ready);
          }
          acc = 1;
          __syncwarp();
          if (!warp_wait(bnd_done, bnd_cnt & 1, lim, abort_flag)) return false;
          tc_fence_after();
          ++bnd_cnt;
          prev = W;
        }
      }
      if (leader) {
        const uint32_t full = pw_full(w);
#pragma unroll
        for (int g = 0; g < G; ++g)
          if ((full >> g) & 1u) {
            umma_ss(s_col, k_desc + g * GD128, qst + g * GD64, IDESC_S, acc);
            acc = 1;
          }
        const uint64_t dost = do_desc + ((st * L::STAGE) >> 4);
#pragma unroll
        for (int g = 0; g < G; ++g)
          umma_ss(tmem + KV_DP, v_desc + g * GD128, dost + g * GD64, IDESC_S, g > 0 ? 1u : 0u);
        umma_commit(s_ready);
      }
      __syncwarp();
      return true;
    };
    // dK[groups] += dS^T Q[groups], one product set per run of consecutive groups
    auto issue_dk_groups = [&](int u, uint32_t groups) {
      const int st = u % TNST;
      const uint64_t qst = qmn_desc + ((st * L::STAGE) >> 4);
      const uint32_t ob = tmem + KV_OB + 64 * (u & 1) + 32;  // dS^T
      while (groups) {
        const int g0 = __ffs(groups) - 1;
        int g1 = g0;
        while (g1 < G && ((groups >> g1) & 1u)) ++g1;
        groups &= ~(((1u << g1) - 1u) & ~((1u << g0) - 1u));
        const uint32_t idesc = idesc_bf16_f32(128, 16 * (g1 - g0), false, true);
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < TBS / 16; ++kk)
            umma_ts(tmem + KV_DK + 16 * g0, ob + 8 * kk, qst + g0 * GD64 + ((kk * 16 * 32) >> 4), idesc, 1u);
        }
        __syncwarp();
      }
    };
    // dV(u), then dK(u): full groups on dS^T as it is, then the boundary
    // classes in descending cutoff order, each after the row warps masked dS^T
    auto issue_dkdv = [&](int u) -> bool {
      const int st = u % TNST;
      const uint32_t w = plans[2 * st];
      const int32_t *cut = cuts + 8 * static_cast<int>(plans[2 * st + 1]);
      if (leader) {
        constexpr uint32_t IDESC_DV = idesc_bf16_f32(128, D, false, true);
        const uint64_t dost = domn_desc + ((st * L::STAGE) >> 4);
        const uint32_t ob = tmem + KV_OB + 64 * (u & 1);  // P^T
#pragma unroll
        for (int kk = 0; kk < TBS / 16; ++kk)
          umma_ts(tmem + L::DV_COL, ob + 8 * kk, dost + ((kk * 16 * 32) >> 4), IDESC_DV, 1u);
      }
      __syncwarp();
      issue_dk_groups(u, pw_full(w));
      int64_t prev = INT64_MAX;
      int32_t W;
      uint32_t cls;
      while (prev_boundary_class(cut, pw_bnd(w), prev, &W, &cls)) {
        if (leader) umma_commit(dsm_req);
        __syncwarp();
        if (!warp_wait(dsm_done, dsm_cnt & 1, lim, abort_flag)) return false;
        tc_fence_after();
        ++dsm_cnt;
        issue_dk_groups(u, cls);
        prev = W;
      }
      if (leader) {
        umma_commit(&qd_empty[st]);
        umma_commit(&ob_free[u & 1]);
      }
      __syncwarp();
      return true;
    };
    // S^T(v + 1) once the row warps have loaded S^T(v)
    auto next_sdp = [&](int v) -> bool {
      uint32_t w;
      if (!warp_wait(s_free, v & 1, lim, abort_flag) || !plan(v + 1, w)) return false;
      return issue_sdp(v + 1, w);
    };

    if (ok && nsub > 0) {
      uint32_t w;
      ok = plan(0, w) && issue_sdp(0, w);
    }
    for (int u = 0; ok && u < nsub; ++u) {
      // S(u + 1) overlaps the row warps' work on u, unless it has boundary
      // classes: then its handshakes follow dK(u) and the row warps' masking for u
      bool early = false;
      if (u + 1 < nsub) {
        uint32_t w1;
        if (!plan(u + 1, w1)) {
          ok = false;
          break;
        }
        if (pw_bnd(w1) == 0u) {
          early = true;
          if (!(ok = next_sdp(u))) break;
        }
      }
      if (!warp_wait(&ds_ready[u & 1], (u >> 1) & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      ok = issue_dkdv(u);
      if (ok && u + 1 < nsub && !early) ok = next_sdp(u);
    }
    if (leader) {
      umma_commit(kv_final);
      umma_commit(drain);
    }
    __syncwarp();
    warp_wait(drain, 0, lim, nullptr);
  } else if (warp < NROWW) {
    // ---------------------------------------------------------- row warps
    const int q4 = warp & 3, cq = warp >> 2, cb = COLS * cq;  // lane quarter, first column
    const int r = q4 * 32 + lane;
    const int64_t j = static_cast<int64_t>(kb) * TBQ + r;  // this thread's key
    const bool row_ok = j < N;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const uint32_t s_addr = lane_addr + KV_S + cb, dp_addr = lane_addr + KV_DP + cb;
    const uint64_t c2x2 = pack_f2(a.scale_log2, a.scale_log2);
    constexpr int DPW = D / CSPLIT;  // accumulator columns of this warp in the epilogue
    tmem_zero16(lane_addr + KV_DK + cq * DPW, DPW / 16);
    tmem_zero16(lane_addr + L::DV_COL + cq * DPW, DPW / 16);
    int bnd_cnt = 0, dsm_cnt = 0;
    bool ok = true;
    for (int u = 0; ok && u < nsub; ++u) {
      const int st = u % TNST;
      const int64_t q0 = q0_of(u) + cb;  // query of my first column
      const uint32_t pt_addr = lane_addr + KV_OB + 64 * (u & 1) + (COLS / 2) * cq, dst_addr = pt_addr + 32;
      if (!warp_wait(&qd_full[st], (u / TNST) & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      const uint32_t w = plans[2 * st];
      const int32_t *cut = cuts + 8 * static_cast<int>(plans[2 * st + 1]);
      if (pw_bnd(w)) {
        // S^T masked in place after each boundary class: keep query c iff (q0 + c) - j <= W
        int64_t prev = -1;
        int32_t W;
        uint32_t cls;
        while (next_boundary_class(cut, pw_bnd(w), prev, &W, &cls)) {
          ok = warp_wait(bnd_ready, bnd_cnt & 1, lim, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const int64_t cm = j - q0 + W;
          const int cmax = cm < -1 ? -1 : (cm > COLS - 1 ? COLS - 1 : static_cast<int>(cm));
          uint32_t su[COLS];
          ld_cols(s_addr, su);
#pragma unroll
          for (int c = 0; c < COLS; ++c)
            if (c > cmax) su[c] = 0u;
          st_cols(s_addr, su);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bnd_done);
          ++bnd_cnt;
          prev = W;
        }
        if (!ok) break;
      }
      // a sleeping poll: a spinning row warp would take issue slots from the
      // MMA warp that shares its scheduler, which is what S(u) waits for
      if (!warp_wait_idle<32>(s_ready, u & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // No S product for this sub-tile: its S is 0. Store the zeros into this
      // warp's S columns (no MMA reads them) so that every sub-tile takes the
      // same loads; zeroing the registers on that path instead gives them two
      // definitions, and the merge costs register moves on every sub-tile.
      if (!(pw_full(w) | pw_bnd(w))) tmem_zero16(s_addr, COLS / 16);
      uint32_t su[COLS], dp[COLS];
      ld_cols2(s_addr, su, dp_addr, dp);
      // S^T and dP^T are in registers: the buffer is free for S^T(u + 1)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);
      // P^T = exp2(S^T c2 - LSE_i log2 e) on the causal pairs i >= j of valid
      // queries, dS^T = P^T (dP^T - D_i)
      const float4 *ld4 = reinterpret_cast<const float4 *>(smem + L::LD_OFF + st * 512) + cq * (COLS / 4);
      const int64_t cm0 = j - q0, cv = N - 1 - q0;  // my first causal and last valid column
      const int lo = !row_ok ? COLS : (cm0 < 0 ? 0 : (cm0 > COLS ? COLS : static_cast<int>(cm0)));
      const int hi = cv > COLS - 1 ? COLS - 1 : static_cast<int>(cv);
      float pf[COLS], ds[COLS];
#pragma unroll
      for (int c4 = 0; c4 < COLS / 4; ++c4) {
        const float4 l4 = ld4[c4], d4 = ld4[16 + c4];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = 4 * c4 + 2 * e;
          const float la = (e == 0 ? l4.x : l4.z) * TLOG2E, lb = (e == 0 ? l4.y : l4.w) * TLOG2E;
          const float da = e == 0 ? d4.x : d4.z, db = e == 0 ? d4.y : d4.w;
          const uint64_t x2 = ffma2(pack_f2(__uint_as_float(su[c]), __uint_as_float(su[c + 1])), c2x2,
                                    pack_f2(-la, -lb));
          float x0, x1;
          unpack_f2(x2, x0, x1);
          const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
          const uint64_t g2 = fsub2(pack_f2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])), pack_f2(da, db));
          float d0, d1;
          unpack_f2(fmul2(pack_f2(p0, p1), g2), d0, d1);
          pf[c] = p0;
          pf[c + 1] = p1;
          ds[c] = d0;
          ds[c + 1] = d1;
        }
      }
      // operand buffer u & 1 is free once the products of u - 2 have read it
      if (u >= 2 && !warp_wait(&ob_free[u & 1], ((u >> 1) - 1) & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      store_bf16_cols(pt_addr, pf, lo, hi);
      store_bf16_cols(dst_addr, ds, lo, hi);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ds_ready[u & 1]);
      int64_t prev = INT64_MAX;
      int32_t W;
      uint32_t cls;
      while (prev_boundary_class(cut, pw_bnd(w), prev, &W, &cls)) {
        ok = warp_wait(dsm_req, dsm_cnt & 1, lim, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const int64_t cm = j - q0 + W;
        const int cmax = cm < -1 ? -1 : (cm > COLS - 1 ? COLS - 1 : static_cast<int>(cm));
        store_bf16_cols(dst_addr, ds, lo, hi < cmax ? hi : cmax);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dsm_done);
        ++dsm_cnt;
        prev = W;
      }
    }
    __nv_bfloat16 *dkrow = a.dk + ((static_cast<int64_t>(b) * a.N + j) * a.Hkv + hk) * D + cq * DPW;
    __nv_bfloat16 *dvrow = a.dv + ((static_cast<int64_t>(b) * a.N + j) * a.Hkv + hk) * D + cq * DPW;
    if (ok && nsub > 0 && warp_wait(kv_final, 0, lim, abort_flag)) {
      tc_fence_after();
      for (int c = 0; c < DPW / 16; ++c) {
        store_row16(lane_addr + KV_DK + cq * DPW + 16 * c, a.scale, dkrow + 16 * c, row_ok);
        store_row16(lane_addr + L::DV_COL + cq * DPW + 16 * c, 1.f, dvrow + 16 * c, row_ok);
      }
    } else {
      *abort_flag = 1;
      if (row_ok) {
        store_nan(dkrow, DPW);
        store_nan(dvrow, DPW);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == T_MMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
cudaError_t launch_dq(const BackwardArgs &a, const BackwardMaps &m, cudaStream_t stream) {
  // one CTA per SM: the kernel holds all 512 TMEM columns
  const uint32_t smem = DqTL<D>::BYTES > 120u * 1024u ? DqTL<D>::BYTES : 120u * 1024u;
  cudaError_t e = cudaFuncSetAttribute(dq_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dq_tc_kernel<D><<<dim3((a.N + TBQ - 1) / TBQ, a.Hq, a.B), TC_THREADS, smem, stream>>>(m.q128, m.do128, m.k64,
                                                                                       m.v64, a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_dkdv(const BackwardArgs &a, const BackwardMaps &m, cudaStream_t stream) {
  const uint32_t smem = KvTL<D>::BYTES > 120u * 1024u ? KvTL<D>::BYTES : 120u * 1024u;
  cudaError_t e = cudaFuncSetAttribute(dkdv_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dkdv_tc_kernel<D><<<dim3((a.N + TBQ - 1) / TBQ, a.Hkv, a.B), TC_THREADS, smem, stream>>>(m.k128, m.v128, m.q64,
                                                                                         m.do64, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_backward_dq_tc(int d_h, const BackwardArgs &a, const BackwardMaps &maps, cudaStream_t stream) {
  return d_h == 128 ? launch_dq<128>(a, maps, stream) : launch_dq<64>(a, maps, stream);
}

cudaError_t launch_backward_dkdv_tc(int d_h, const BackwardArgs &a, const BackwardMaps &maps, cudaStream_t stream) {
  return d_h == 128 ? launch_dkdv<128>(a, maps, stream) : launch_dkdv<64>(a, maps, stream);
}

}  // namespace wp
