// WavePrune grouped-cutoff causal prefill on sm_100a: TMA + tcgen05 + TMEM.
//
// What it computes (WavePrune reading notes "WavePrune：RoPE 通常只需一个旋转
// 周期", §2.1 Eq. (6) and §2.3 Eq. (8)): for j <= i,
//   L_ij = scale * sum_g 1[i - j <= W_g] * (Q_i[16g:16g+16] . K_j[16g:16g+16]),
// then the usual causal softmax and O = A V. A masked group adds 0 to the
// logit (detail 1 of §2.1), the pair stays in the softmax.
//
// How. One CTA takes one 128-row query tile of two query heads that share a
// KV head (GQA), so every K/V tile it loads feeds both, and visits the key
// tiles from the diagonal backwards. Each 128-key tile is handled as two
// 64-key sub-tiles u = 2t + h; §2.3's skip / full / boundary class of
// every (sub-tile, group) comes from a per-CTA table built once in shared
// memory (one table for both heads, or one per head when each query head has
// its own cutoff table).
//   warp 8   TMA producer: Q of both heads once (one 16-dim box per group);
//            per key tile only the K column slices of groups either half
//            (of either head) computes (16-dim boxes, 32-byte swizzle) and all of V (64-dim
//            boxes, 128-byte swizzle); two stages each.
//   warp 9+s MMA issuer of head s (one elected lane, warp-uniform loop). S of
//            a head is double-buffered: two 64-column halves of TMEM, half h
//            holding sub-tiles u = h mod 2. Per sub-tile u: once P(u) is in
//            TMEM, PV(u) (4 MMAs, K = 16 keys each, into O) and then QK(u+2)
//            into the half P(u) frees (one M=128, N=64, K=16 MMA per
//            non-skipped group). The tensor core runs one thread's MMAs in
//            order, so QK(u+2) overwrites P(u) only after PV(u) has read it,
//            and S(u+1) was issued one step earlier: the softmax of u+1 runs
//            while the MMAs that follow u do.
//   warps 0-3 / 4-7  softmax of head 0 / head 1, one thread per query row:
//            causal mask on the diagonal tile, online softmax in base 2 with
//            the scale folded into one FMA, P (bf16) over the first 32
//            columns of its S half, O rescaled only when a row max grows by
//            more than 2^8; epilogue O/l -> bf16 and LSE = ln(sum exp).
// Boundary groups: the groups whose cutoff falls inside the sub-tile's
// distance range go first, one distinct cutoff at a time in ascending order;
// after each class the softmax warps mask S in place (keep iff i - j <= W,
// else 0), and the full groups then accumulate on top unmasked. Masks of
// ascending cutoffs are nested, so m2*(m1*S1 + S2) = m1*S1 + m2*S2: the
// exact per-class mask.
// TMEM columns: head s uses [256s, 256s+64) and [256s+64, 256s+128) for the
// two S / P halves and [256s+128, 256s+256) for O. If H_q/H_kv is odd the CTA
// takes a single head.
//
// The softmax's exponentials compete with the MUFU unit's 16 per SM per
// clock, so POLY_PAIRS of every 8 pairs take 2^x on the FMA pipe instead, in
// packed f32x2 arithmetic: Cody-Waite reduction x = j + f, |f| <= 1/2, and a
// degree-3 minimax polynomial for 2^f (coefficients from a Remez fit, max
// relative error 7.5e-5, far below bf16's 2^-9 for P), scaled by 2^j in the
// exponent field. The diagonal tile takes every exponential on MUFU, so its
// causally masked entries give exactly 0.
//
// Packed (varlen) batches: sequence b occupies rows cu_seqlens[b] ..
// cu_seqlens[b+1]-1 of [T, H, d]; positions restart at 0 in every sequence.
// A tile that runs past the sequence's end loads the next rows of the buffer,
// which only the diagonal tile's causal mask ever sees (P exactly 0).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <type_traits>

#include "wp_device.cuh"
#include "wp_prefill.h"
#include "wp_prefill_common.cuh"
#include "wp_tile.h"

namespace wp {

namespace {

constexpr int BM = 128;
constexpr int BN = 128;   // key tile of the K/V loads
constexpr int SUB = 64;   // key sub-tile of one S buffer (two per head, double-buffered)
constexpr int KST = 2;  // K stages
constexpr int VST = 2;  // V stages
constexpr int NTHREADS = 352;  // warps 0-7 softmax (2 heads), 8 TMA producer, 9/10 MMA issuer of head 0/1
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;  // head s is issued by warp MMA_WARP + s; this one also owns TMEM
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t GROUP_TILE_BYTES = 128 * 32;  // 128 rows x 16 bf16
constexpr uint32_t V_CHUNK_BYTES = 128 * 128;    // 128 keys x 64 bf16

__host__ __device__ constexpr uint32_t col_s(int slot) { return 256u * slot; }
__host__ __device__ constexpr uint32_t col_o(int slot) { return 256u * slot + 128u; }

template <int D>
struct Layout {
  static constexpr int G = D / 16;
  static constexpr uint32_t Q_SLOT = G * GROUP_TILE_BYTES;
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t K_OFF = Q_OFF + 2 * Q_SLOT;
  static constexpr uint32_t K_STAGE = G * GROUP_TILE_BYTES;
  static constexpr uint32_t V_OFF = K_OFF + KST * K_STAGE;
  static constexpr uint32_t V_STAGE = (D / 64) * V_CHUNK_BYTES;
  static constexpr uint32_t BAR_OFF = V_OFF + VST * V_STAGE;
  // q_full, k_full/empty, v_full/empty, per head x half s_ready/p_ready, per head
  // o_ready/o_final/bnd_ready/bnd_done, drain
  static constexpr uint32_t NUM_BARS = 1 + 2 * KST + 2 * VST + 2 * 4 + 2 * 4 + 2;
  static constexpr uint32_t MISC_OFF = BAR_OFF + NUM_BARS * 8;
  static constexpr uint32_t CUT_OFF = MISC_OFF + 16;  // cutoff rows of head slot 0 and 1: 2 x 8 int32
  static constexpr uint32_t TT_OFF = CUT_OFF + 64;    // sub-tile tables: one uint16 per 64-key sub-tile
  // One table per head slot when the two heads have their own cutoffs, one
  // shared table otherwise.
  static uint32_t table_bytes(int nqb, bool per_head) { return ((4u * nqb + 15u) & ~15u) * (per_head ? 2u : 1u); }
  static uint32_t bytes(int nqb, bool per_head) { return TT_OFF + table_bytes(nqb, per_head) + 1024u; }  // + align
};

struct Barriers {
  uint64_t *q_full, *k_full, *k_empty, *v_full, *v_empty, *s_ready, *p_ready, *o_ready, *o_final, *bnd_ready,
      *bnd_done, *drain;
};

// The per-head cutoff parameter of a kernel instantiation: the table, or a
// placeholder when every head shares the table in PrefillArgs.
struct NoHeadCuts {
  int32_t unused;
};
template <bool PER_HEAD>
using HeadCutsArg = typename std::conditional<PER_HEAD, HeadCuts, NoHeadCuts>::type;

// Class masks of the 128-query x 64-key block (qb, kb64) under the cutoff
// row `cut` (shared memory): bits 0-7 full groups, bits 8-15 boundary groups.
__device__ __forceinline__ uint32_t sub_masks(const int32_t *cut, int G, int64_t N, int64_t qb, int64_t kb64) {
  int64_t dmin = 0, dmax = -1;
  uint32_t full = 0, bnd = 0;
  if (tile_distance_range(N, BM, SUB, qb, kb64, &dmin, &dmax)) {
    for (int g = 0; g < G; ++g) {
      const int c = classify_cutoff(dmin, dmax, cut[g]);
      if (c == TILE_FULL) full |= 1u << g;
      if (c == TILE_BOUNDARY) bnd |= 1u << g;
    }
  }
  return full | (bnd << 8);
}

// PACKED: sequences located by cu_seqlens (else a uniform batch); PER_HEAD:
// one cutoff row per query head (else one row for all). Both are template
// parameters so that the plain case carries none of their bookkeeping.
template <int D, bool PACKED, bool PER_HEAD>
__global__ void __launch_bounds__(NTHREADS, 1)
    prefill_grouped_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const PrefillArgs a,
                           const HeadCutsArg<PER_HEAD> hc) {
  using L = Layout<D>;
  constexpr int G = L::G;
  constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, SUB, false, false);
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
  B.s_ready = B.v_empty + VST;  // [2 heads][2 halves]
  B.p_ready = B.s_ready + 4;    // [2 heads][2 halves]
  B.o_ready = B.p_ready + 4;
  B.o_final = B.o_ready + 2;  // completes once, after the last PV of the head
  B.bnd_ready = B.o_final + 2;
  B.bnd_done = B.bnd_ready + 2;
  B.drain = B.bnd_done + 2;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::MISC_OFF);
  uint32_t *tmem_base_slot = reinterpret_cast<uint32_t *>(smem + L::MISC_OFF + 4);
  // Sub-tile class tables of head slot 0 and 1 (the same table unless the
  // heads have their own cutoffs).
  uint16_t *ttab0 = reinterpret_cast<uint16_t *>(smem + L::TT_OFF);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  // Grid (head pair within its KV group, query block, KV head x batch): the
  // CTAs that run together share one KV head, so its K/V stay in L2; within
  // a KV head the heaviest query blocks go first.
  const int rep = a.Hq / a.Hkv;
  const int nslot = (rep % 2 == 0) ? 2 : 1;
  const int hk = static_cast<int>(blockIdx.z) % a.Hkv;
  const int b = static_cast<int>(blockIdx.z) / a.Hkv;
  const int h0 = hk * rep + static_cast<int>(blockIdx.x) * nslot;  // head of slot s = h0 + s
  const int nqb = (a.N + BM - 1) / BM;
  const int qb = nqb - 1 - static_cast<int>(blockIdx.y);
  // The sequence: batch entry b of a uniform batch (length a.N, coordinate b
  // of the 4-D tensor view) or rows [row0, row0 + N) of a packed one.
  int64_t N = a.N, row0 = 0;
  if constexpr (PACKED) {
    row0 = a.cu_seqlens[b];
    const int64_t row1 = a.cu_seqlens[b + 1];
    if (row0 < 0 || row1 < row0 || row1 > a.T || row1 - row0 > a.N) {
      // Offsets out of range: nothing of this sequence can be located.
      if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0 && hk == 0) record_status(WP_ERR_ARG);
      return;
    }
    N = row1 - row0;
    if (static_cast<int64_t>(qb) * BM >= N) return;  // past this sequence's end (whole CTA)
  }
  // TMA row coordinate of query / key block x and the batch coordinate
  const auto block_row = [&](int x) { return PACKED ? static_cast<int>(row0 + static_cast<int64_t>(x) * BM) : x * BM; };
  const int bcoord = PACKED ? 0 : b;
  // the cutoff rows of head slot 0 and 1, copied into shared memory below
  int32_t *cut0 = reinterpret_cast<int32_t *>(smem + L::CUT_OFF);
  int32_t *cut1 = PER_HEAD ? cut0 + 8 : cut0;
  uint16_t *ttab1 = PER_HEAD ? ttab0 + ((2 * qb + 2 + 7) & ~7) : ttab0;
  const long long lim = a.wait_limit;

  if (threadIdx.x == 0) {
    // A kernel of this library has given up since the status word was last
    // read (this call or an earlier one): skip the work and write NaN rows.
    *abort_flag = *reinterpret_cast<volatile int *>(&g_status) != 0 ? 1 : 0;
    mbar_init(B.q_full, 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(&B.k_full[s], 1);
      mbar_init(&B.k_empty[s], nslot);  // one commit per head's MMA warp
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(&B.v_full[s], 1);
      mbar_init(&B.v_empty[s], nslot);
    }
    for (int s = 0; s < 4; ++s) {
      mbar_init(&B.s_ready[s], 1);
      mbar_init(&B.p_ready[s], 4);  // one arrival per softmax warp
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&B.o_ready[s], 1);
      mbar_init(&B.o_final[s], 1);
      mbar_init(&B.bnd_ready[s], 1);
      mbar_init(&B.bnd_done[s], 4);
    }
    mbar_init(&B.drain[0], 1);
    mbar_init(&B.drain[1], 1);
    fence_barrier_init();
  }
  if (threadIdx.x == 0) {  // the cutoff rows of both head slots (constant indices into the parameters)
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      if constexpr (PER_HEAD) {
        cut0[g] = g < G ? hc.cut[h0 * G + g] : WP_CUTOFF_INF;
        cut0[8 + g] = g < G ? hc.cut[(h0 + nslot - 1) * G + g] : WP_CUTOFF_INF;
      } else {
        cut0[g] = a.cut[g];
      }
    }
  }
  __syncthreads();
  // Sub-tile table: sub-tile u = 2t + h holds the keys of 64-key block
  // 2(qb - t) + h, i.e. half h of key tile t.
  for (int u = threadIdx.x; u < 2 * (qb + 1); u += NTHREADS) {
    const int64_t kb64 = 2 * (qb - u / 2) + (u & 1);
    ttab0[u] = static_cast<uint16_t>(sub_masks(cut0, G, N, qb, kb64));
    if (PER_HEAD) ttab1[u] = static_cast<uint16_t>(sub_masks(cut1, G, N, qb, kb64));
  }
  if (warp == MMA_WARP) {
    tmem_alloc(tmem_base_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_slot;
  const int nkb = *abort_flag ? 0 : qb + 1;  // key tiles qb, qb-1, ..., 0 (BM == BN)
  const int nsub = 2 * nkb;

  if (warp == PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the loop (warp-uniform waits); one elected lane
    // issues each bulk copy.
    const bool leader = elect_one();
    const int qrow = block_row(qb);
    if (leader) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(B.q_full, nslot * G * GROUP_TILE_BYTES);
      for (int s = 0; s < nslot; ++s)
        for (int g = 0; g < G; ++g)
          tma_load_4d(smem + L::Q_OFF + s * L::Q_SLOT + g * GROUP_TILE_BYTES, &tm_q, B.q_full, 16 * g, h0 + s, qrow,
                      bcoord);
    }
    __syncwarp();
    int k_issued = 0, v_issued = 0;
    bool ok = true;
    auto load_v = [&](int t) -> bool {
      const int st = t % VST;
      if (t >= VST && !warp_wait_idle(&B.v_empty[st], ((t / VST) - 1) & 1, lim, abort_flag)) return false;
      const int krow = block_row(qb - t);
      if (leader) {
        mbar_arrive_expect_tx(&B.v_full[st], (D / 64) * V_CHUNK_BYTES);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(smem + L::V_OFF + st * L::V_STAGE + c * V_CHUNK_BYTES, &tm_v, &B.v_full[st], 64 * c, hk, krow,
                      bcoord);
      }
      __syncwarp();
      ++v_issued;
      return true;
    };
    for (int t = 0; ok && t < nkb; ++t) {
      const int st = t % KST;
      if (t >= KST && !warp_wait_idle(&B.k_empty[st], ((t / KST) - 1) & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      const int krow = block_row(qb - t);
      // groups either half of the tile computes, for either head
      const uint32_t m =
          ttab0[2 * t] | ttab0[2 * t + 1] | (PER_HEAD && nslot == 2 ? ttab1[2 * t] | ttab1[2 * t + 1] : 0u);
      const uint32_t need = (m | (m >> 8)) & 0xffu;
      if (leader) {
        mbar_arrive_expect_tx(&B.k_full[st], __popc(need) * GROUP_TILE_BYTES);
        for (uint32_t mm = need; mm; mm &= mm - 1) {
          const int g = __ffs(mm) - 1;
          tma_load_4d(smem + L::K_OFF + st * L::K_STAGE + g * GROUP_TILE_BYTES, &tm_k, &B.k_full[st], 16 * g, hk,
                      krow, bcoord);
        }
      }
      __syncwarp();
      ++k_issued;
      if (t >= 1) ok = load_v(t - 1);
    }
    if (ok && nkb >= 1) ok = load_v(nkb - 1);
    // Never leave a bulk copy in flight into shared memory this CTA is about
    // to release: wait for Q and the last issued load of every stage.
    warp_wait_idle(B.q_full, 0, lim, nullptr);
    for (int s = 0; s < KST && s < k_issued; ++s) {
      const int last = s + ((k_issued - 1 - s) / KST) * KST;
      warp_wait_idle(&B.k_full[s], (last / KST) & 1, lim, nullptr);
    }
    for (int s = 0; s < VST && s < v_issued; ++s) {
      const int last = s + ((v_issued - 1 - s) / VST) * VST;
      warp_wait_idle(&B.v_full[s], (last / VST) & 1, lim, nullptr);
    }
  } else if (warp >= MMA_WARP && warp < MMA_WARP + nslot) {
    // ------------------------------------------------------- MMA issuers
    // Warp MMA_WARP + s issues head slot s: the whole warp runs the issue
    // loop (control flow and descriptors are warp-uniform) and one elected
    // lane issues each group of tcgen05.mma / commit in one branch. The two
    // heads' loops run side by side; tcgen05.commit tracks the MMAs of the
    // issuing thread only, so each head's barriers see its own MMAs.
    const int s = warp - MMA_WARP;
    const bool leader = elect_one();
    // Descriptor bases; a byte offset within shared memory is added to the
    // start-address field (bits 0-13, in 16-byte units).
    const uint64_t q_desc = smem_desc(smem_u32(smem + L::Q_OFF), 16, 256, SMEM_SWIZZLE_32B);
    const uint64_t k_desc = smem_desc(smem_u32(smem + L::K_OFF), 16, 256, SMEM_SWIZZLE_32B);
    // V tile: 128 keys x D, dims contiguous (MN-major), 128-byte swizzle;
    // 8-key row groups 1024 B apart, 64-dim chunks 16 KB apart.
    const uint64_t v_desc = smem_desc(smem_u32(smem + L::V_OFF), V_CHUNK_BYTES, 1024, SMEM_SWIZZLE_128B);
    int bnd_cnt = 0;
    bool ok = warp_wait(B.q_full, 0, lim, abort_flag);

    // One MMA (M=128, N=64, K=16) per group of `groups`, accumulating after
    // the first.
    auto issue_groups = [&](uint32_t s_col, uint64_t qs_desc, uint64_t kst_desc, uint32_t groups, uint32_t acc) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        if (groups & (1u << g)) {
          umma_ss(s_col, qs_desc + g * (GROUP_TILE_BYTES >> 4), kst_desc + g * (GROUP_TILE_BYTES >> 4), IDESC_QK,
                  acc);
          acc = 1;
        }
      }
    };
    // QK of this head for sub-tile u into S half u & 1 (its K stage loaded).
    const uint16_t *ttab = s == 0 ? ttab0 : ttab1;
    const int32_t *cut = s == 0 ? cut0 : cut1;
    auto issue_qk = [&](int u) -> bool {
      const uint32_t tm = ttab[u];
      const int t = u >> 1, hh = u & 1;
      const uint32_t s_col = tmem + col_s(s) + SUB * hh;
      const uint64_t qs_desc = q_desc + ((s * L::Q_SLOT) >> 4);
      // key rows 64*hh.. of every K group tile (32 bytes per row)
      const uint64_t kst_desc = k_desc + (((t % KST) * L::K_STAGE + hh * SUB * 32) >> 4);
      uint32_t acc = 0;
      const uint32_t bnd = tm >> 8;
      if (bnd) {
        // boundary classes first, ascending cutoff; each one masked in place
        int64_t prev = -1;
        int32_t W;
        uint32_t cls;
        while (next_boundary_class(cut, bnd, prev, &W, &cls)) {
          if (leader) {
            issue_groups(s_col, qs_desc, kst_desc, cls, acc);
            umma_commit(&B.bnd_ready[s]);
          }
          acc = 1;
          __syncwarp();
          if (!warp_wait(&B.bnd_done[s], bnd_cnt & 1, lim, abort_flag)) return false;
          tc_fence_after();
          ++bnd_cnt;
          prev = W;
        }
      }
      if (leader) {
        issue_groups(s_col, qs_desc, kst_desc, tm & 0xffu, acc);
        umma_commit(&B.s_ready[2 * s + hh]);
      }
      __syncwarp();
      return true;
    };

    if (ok && nkb > 0) {
      ok = warp_wait(&B.k_full[0], 0, lim, abort_flag);
      if (ok) {
        tc_fence_after();
        ok = issue_qk(0);
        if (ok) ok = issue_qk(1);
        if (ok && leader) umma_commit(&B.k_empty[0]);
        __syncwarp();
      }
    }
    // Per sub-tile u and head: PV(u) as soon as P(u) is in TMEM, then
    // QK(u + 2) into the S half that P(u) frees (the tensor core runs them in
    // order); S(u + 1) was issued one step earlier, so the softmax never
    // waits for the MMAs that follow its own P.
    for (int u = 0; ok && u < nsub; ++u) {
      const int t = u >> 1, hh = u & 1;
      const int vst = t % VST;
      if (hh == 0 && !warp_wait(&B.v_full[vst], (t / VST) & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      const uint64_t vst_desc = v_desc + ((vst * L::V_STAGE) >> 4);
      // one barrier per S half: the softmax of the other half may already
      // have arrived for the next sub-tile
      if (!warp_wait(&B.p_ready[2 * s + hh], t & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t p_col = tmem + col_s(s) + SUB * hh;
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < SUB / 16; ++kk)
          umma_ts(tmem + col_o(s), p_col + kk * 8, vst_desc + (hh * (SUB / 16) + kk) * (2048 >> 4), IDESC_PV,
                  (u > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&B.o_ready[s]);
        if (u == nsub - 1) umma_commit(&B.o_final[s]);
        if (hh == 1) umma_commit(&B.v_empty[vst]);
      }
      __syncwarp();
      if (u + 2 < nsub) {
        if (hh == 0) {
          // QK(u + 2) opens key tile t + 1
          if (!warp_wait(&B.k_full[(t + 1) % KST], ((t + 1) / KST) & 1, lim, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        ok = issue_qk(u + 2);
        if (ok && hh == 1) {
          // QK(u + 2) closed key tile t + 1
          if (leader) umma_commit(&B.k_empty[(t + 1) % KST]);
          __syncwarp();
        }
      }
    }
    // Every MMA this warp issued must finish before TMEM is released.
    if (leader) umma_commit(&B.drain[s]);
    __syncwarp();
    warp_wait(&B.drain[s], 0, lim, nullptr);
  } else if (warp / 4 < nslot) {
    // ------------------------------------------------------- softmax warps
    // Every tcgen05.ld/st/wait below is .sync.aligned: the whole warp must
    // issue it together. So every wait is made warp-uniform (warp_wait), the
    // O-rescale decision is a warp vote, and only the global stores of the
    // padding rows of a ragged last tile are predicated.
    const int slot = warp / 4;
    const int q4 = warp % 4;
    const int r = q4 * 32 + lane;  // row of the query tile == TMEM lane
    const int h = h0 + slot;
    const uint16_t *ttab = slot == 0 ? ttab0 : ttab1;
    const int32_t *cut = slot == 0 ? cut0 : cut1;
    const int64_t i = static_cast<int64_t>(qb) * BM + r;  // position in the sequence
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const uint32_t o_addr = lane_addr + col_o(slot);
    const float c2 = a.scale_log2;  // logits to base-2 exponent units
    const uint64_t c2x2 = pack_f2(c2, c2);
    float m_run = -INFINITY, l_run = 0.f;  // running max (base-2 units) and sum
    int bnd_cnt = 0;
    bool ok = true;
    for (int u = 0; u < nsub; ++u) {
      const int t = u >> 1, hh = u & 1;
      const int64_t k0 = static_cast<int64_t>(qb - t) * BN + SUB * hh;  // first key of the sub-tile
      const uint32_t s_addr = lane_addr + col_s(slot) + SUB * hh;
      const uint32_t tm = ttab[u];
      const uint32_t bnd = tm >> 8;
      const bool any_group = (tm & 0xffffu) != 0;
      if (bnd) {
        // Mask S in place after each boundary class: keep column c iff
        // (i - k0) - c <= W, i.e. c >= cmin; otherwise 0.
        int64_t prev = -1;
        int32_t W;
        uint32_t cls;
        while (next_boundary_class(cut, bnd, prev, &W, &cls)) {
          ok = warp_wait(&B.bnd_ready[slot], bnd_cnt & 1, lim, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const int64_t cmin64 = i - k0 - W;
          const int cmin = cmin64 < 0 ? 0 : (cmin64 > SUB ? SUB : static_cast<int>(cmin64));
          uint32_t su[64];
          tmem_ld64(s_addr, su);
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c < cmin) su[c] = 0u;
          tmem_st32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&su[0]));
          tmem_st32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&su[32]));
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&B.bnd_done[slot]);
          ++bnd_cnt;
          prev = W;
        }
        if (!ok) break;
      }
      if (!warp_wait(&B.s_ready[2 * slot + hh], t & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t su[64];
      load_half(s_addr, any_group, su);
      if (t == 0) causal_mask(su, SUB * hh, r);  // diagonal tile
      const float m_half = half_max(su) * c2;    // scale > 0, so the max commutes with it
      if (u == 0) {
        m_run = m_half;  // key 0 of the diagonal tile is in every row's window
      } else if (__any_sync(FULL, m_half > m_run + RESCALE_THRESHOLD)) {
        // Some row's max grew by more than 2^8 (rare): rescale O (it holds the
        // sum through sub-tile u - 1: wait for that PV) and the row sum.
        const float m_new = fmaxf(m_run, m_half);
        const float alpha = fast_exp2(m_run - m_new);
        if (!warp_wait(&B.o_ready[slot], (u - 1) & 1, lim, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        scale_cols_f32(o_addr, D / 32, alpha);
        l_run *= alpha;
        m_run = m_new;
      }
      const uint64_t zero2 = 0ull;
      uint64_t acc[4] = {zero2, zero2, zero2, zero2};
      // P: the sub-tile's first 32 columns. In a packed batch the diagonal
      // tile takes every exponential on MUFU, so its causally masked entries
      // (possibly the next sequence's keys) give exactly 0.
      if (PACKED && t == 0)
        exp_half<false>(su, c2x2, m_run, acc, s_addr);
      else
        exp_half<true>(su, c2x2, m_run, acc, s_addr);
      float s0, s1, s2, s3, s4, s5, s6, s7;
      unpack_f2(acc[0], s0, s1);
      unpack_f2(acc[1], s2, s3);
      unpack_f2(acc[2], s4, s5);
      unpack_f2(acc[3], s6, s7);
      l_run += ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();  // the warp's TMEM stores are ordered before lane 0's arrival
      if (lane == 0) mbar_arrive(&B.p_ready[2 * slot + hh]);
    }
    __nv_bfloat16 *orow = a.o + (((PACKED ? row0 : static_cast<int64_t>(b) * a.N) + i) * a.Hq + h) * D;
    float *lse_at = a.lse == nullptr
                        ? nullptr
                        : a.lse + (PACKED ? static_cast<int64_t>(h) * a.T + row0 + i
                                                           : (static_cast<int64_t>(b) * a.Hq + h) * a.N + i);
    // o_ready may trail by two phases here (the last two PVs can both be in
    // flight), so the end of the last PV has a barrier of its own.
    if (ok && nsub > 0 && warp_wait(&B.o_final[slot], 0, lim, abort_flag)) {
      tc_fence_after();
      const float inv_l = 1.f / l_run;
#pragma unroll
      for (int c4 = 0; c4 < D / 32; ++c4) {
        uint32_t u32[32];
        tmem_ld32(o_addr + 32 * c4, u32);
        tmem_wait_ld(u32);
        uint4 pk4[4];
        uint32_t *pw = reinterpret_cast<uint32_t *>(pk4);
#pragma unroll
        for (int k = 0; k < 16; ++k)
          pw[k] = pack_bf16x2(__uint_as_float(u32[2 * k]) * inv_l, __uint_as_float(u32[2 * k + 1]) * inv_l);
        if (i < N) {
          uint4 *dst = reinterpret_cast<uint4 *>(orow + 32 * c4);
#pragma unroll
          for (int k = 0; k < 4; ++k) dst[k] = pk4[k];
        }
      }
      if (i < N && lse_at != nullptr) *lse_at = (m_run + log2f(l_run)) * 0.69314718055994531f;
    } else {
      // Tell the other roles to stop waiting for this warp's progress, and
      // never leave the caller's buffers with stale rows: an aborted CTA
      // writes NaN to its O rows and LSE entries.
      *abort_flag = 1;
      if (i < N) {
        const uint4 nan4 = make_uint4(0x7FC07FC0u, 0x7FC07FC0u, 0x7FC07FC0u, 0x7FC07FC0u);
#pragma unroll
        for (int k = 0; k < D / 8; ++k) reinterpret_cast<uint4 *>(orow)[k] = nan4;
        if (lse_at != nullptr) *lse_at = __int_as_float(0x7FC00000);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}
}  // namespace

template <int D, bool PACKED, bool PER_HEAD>
static cudaError_t launch_grouped(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                  const PrefillArgs &a, const HeadCuts *head_cuts, cudaStream_t stream) {
  const int nqb = (a.N + BM - 1) / BM;
  const uint32_t smem = Layout<D>::bytes(nqb, a.cut_rows != 1);
  if (smem > 232448u) return cudaErrorInvalidValue;  // beyond 227 KB: N too large for the tile table
  cudaError_t e = cudaFuncSetAttribute(prefill_grouped_kernel<D, PACKED, PER_HEAD>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int rep = a.Hq / a.Hkv;
  const int nslot = (rep % 2 == 0) ? 2 : 1;
  dim3 grid(rep / nslot, nqb, a.Hkv * a.B);
  HeadCutsArg<PER_HEAD> hc;
  if constexpr (PER_HEAD)
    hc = *head_cuts;
  else
    hc.unused = 0;
  prefill_grouped_kernel<D, PACKED, PER_HEAD><<<grid, NTHREADS, smem, stream>>>(tq, tk, tv, a, hc);
  return cudaGetLastError();
}

cudaError_t launch_prefill_grouped(int d_h, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                   const PrefillArgs &a, const HeadCuts *head_cuts, cudaStream_t stream) {
  const bool packed = a.cu_seqlens != nullptr, per_head = head_cuts != nullptr;
  if (d_h == 128) {
    if (packed) return per_head ? launch_grouped<128, true, true>(tq, tk, tv, a, head_cuts, stream)
                                : launch_grouped<128, true, false>(tq, tk, tv, a, head_cuts, stream);
    return per_head ? launch_grouped<128, false, true>(tq, tk, tv, a, head_cuts, stream)
                    : launch_grouped<128, false, false>(tq, tk, tv, a, head_cuts, stream);
  }
  if (packed) return per_head ? launch_grouped<64, true, true>(tq, tk, tv, a, head_cuts, stream)
                              : launch_grouped<64, true, false>(tq, tk, tv, a, head_cuts, stream);
  return per_head ? launch_grouped<64, false, true>(tq, tk, tv, a, head_cuts, stream)
                  : launch_grouped<64, false, false>(tq, tk, tv, a, head_cuts, stream);
}

}  // namespace wp
