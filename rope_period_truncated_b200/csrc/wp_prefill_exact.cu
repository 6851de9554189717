// WavePrune exact per-channel causal prefill on sm_100a: TMA + tcgen05 + TMEM.
//
// What it computes (WavePrune reading notes "WavePrune：RoPE 通常只需一个旋转
// 周期", §2.1 Eq. (6)): for j <= i,
//   L_ij = scale * sum_c 1[i - j <= W_c] * (q_a k_a + q_b k_b)   (channel c = dims a, b),
// then the causal softmax and O = A V. A dropped channel adds 0; the pair
// stays in the softmax.
//
// How. The grouped kernel's pipeline: one CTA takes one 128-row query tile
// of two query heads that share a KV head; a TMA producer warp, one MMA-issuing
// warp per head, S of each head double-buffered in two 64-key TMEM halves,
// four softmax warps per head with one thread per query row. What changes is
// the logit tile: a tensor-core product covers 16 dims (one group), while the
// rule keeps or drops single channels. For a 64-key sub-tile with distances
// [dmin, dmax], every channel is skip (W_c < dmin), full (W_c >= dmax) or
// boundary; then
//   - a group whose channels are all full is one plain product;
//   - a group with some full channels is one product against a copy of the
//     head's Q slice in which the dims of every other channel are zero. The
//     kept set of a group only changes when a channel's cutoff crosses the
//     tile's distance range, so the head's MMA warp keeps a few such copies
//     in shared memory (TMA layout, fenced for the tensor core's async
//     proxy) and writes a new one only when a new (group, kept set) appears;
//   - a boundary channel's product is rank 2, q_a k_a^T + q_b k_b^T: the
//     softmax threads add it to their row of S with CUDA-core FMAs, only at
//     the keys within W_c of the row, reading Q and K from the tiles the TMA
//     loads already hold (so a K stage with boundary work is free again once
//     the softmax warps are done with it too).
// A plan warp writes each key tile's channel plan (per head when the heads
// have their own cutoffs) into a two-entry ring beside the K stages, ahead of
// the data.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "wp_device.cuh"
#include "wp_prefill.h"
#include "wp_prefill_common.cuh"
#include "wp_tile.h"

namespace wp {

namespace {

constexpr int XBM = 128;
constexpr int XBN = 128;  // key tile of the K/V loads
constexpr int XSUB = 64;  // key sub-tile of one S buffer
constexpr int XKST = 2;
constexpr int XVST = 2;
constexpr int XTHREADS = 384;  // warps 0-7 softmax (2 heads), 8 TMA producer, 9/10 MMA issuer of head 0/1, 11 tile plans
constexpr int XPRODUCER = 8;
constexpr int XMMA = 9;
constexpr int XFINISH = 11;
constexpr uint32_t XTMEM_COLS = 512;
constexpr uint32_t XGROUP_BYTES = 128 * 32;  // 128 rows x 16 bf16
constexpr uint32_t XHALF_BYTES = 64 * 32;    // the 64 keys of one sub-tile
constexpr uint32_t XV_CHUNK = 128 * 128;     // 128 keys x 64 bf16
constexpr int NVAR = 2;    // partially kept groups per sub-tile (masked Q products)
constexpr int QSLOTS = 4;  // masked Q copies kept per head: NVAR for the MMAs in flight, NVAR new

__host__ __device__ constexpr uint32_t xcol_s(int slot) { return 256u * slot; }
__host__ __device__ constexpr uint32_t xcol_o(int slot) { return 256u * slot + 128u; }

template <int D>
struct XLayout {
  static constexpr int G = D / 16;
  static constexpr uint32_t Q_SLOT = G * XGROUP_BYTES;
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t K_OFF = Q_OFF + 2 * Q_SLOT;
  static constexpr uint32_t K_STAGE = G * XGROUP_BYTES;
  static constexpr uint32_t V_OFF = K_OFF + XKST * K_STAGE;
  static constexpr uint32_t V_STAGE = (D / 64) * XV_CHUNK;
  // masked Q copies [head][QSLOTS], one group tile each
  static constexpr uint32_t QV_OFF = V_OFF + XVST * V_STAGE;
  static constexpr uint32_t BAR_OFF = QV_OFF + 2 * QSLOTS * XGROUP_BYTES;
  // q_full, k_full/empty/plan, v_full/empty, per head x half s_ready/p_ready,
  // per head o_ready/o_final/drain
  static constexpr uint32_t NUM_BARS = 1 + 3 * XKST + 2 * XVST + 2 * 4 + 2 * 3;
  static constexpr uint32_t MISC_OFF = BAR_OFF + NUM_BARS * 8;
  static constexpr uint32_t CUT_OFF = MISC_OFF + 16;    // channel cutoffs [plan][64] int32
  static constexpr uint32_t GMAX_OFF = CUT_OFF + 512;   // largest cutoff of each group [plan][8] int32
  static constexpr uint32_t RING_OFF = GMAX_OFF + 64;   // plans [stage][plan][half] x {full, bnd}
  static constexpr uint32_t END = RING_OFF + XKST * 2 * 2 * 16;
  static constexpr uint32_t BYTES = END + 1024;  // + alignment of the dynamic base
};
static_assert(XLayout<128>::BYTES <= PREFILL_SMEM_CAP, "exact prefill layout exceeds shared memory");

// Dims of group g (bit k = dim 16g + k) that belong to the channels in `chans`.
// Interleaved: channel c owns dims 2c, 2c+1, so group g holds channels
// 8g..8g+7, each twice. Half-split: channel c owns dims c and c + D/2, so
// group g holds channels 16 (g mod D/32) .. +15, once each.
template <int D>
__device__ __forceinline__ uint32_t group_keep(uint64_t chans, int g, bool inter) {
  if (inter) {
    uint32_t x = static_cast<uint32_t>(chans >> (8 * g)) & 0xffu;
    x = (x | (x << 4)) & 0x0f0fu;
    x = (x | (x << 2)) & 0x3333u;
    x = (x | (x << 1)) & 0x5555u;
    return x | (x << 1);
  }
  return static_cast<uint32_t>(chans >> (16 * (g % (D / 32)))) & 0xffffu;
}

// Channels owning dims of group g.
template <int D>
__device__ __forceinline__ uint64_t group_chans(int g, bool inter) {
  return inter ? 0xffull << (8 * g) : 0xffffull << (16 * (g % (D / 32)));
}

// Channel plan of the 128-query x 64-key block (qb, kb64), warp-wide: lane l
// classifies channels l and l + 32, and two ballots per class gather the
// masks. `full` channels go to plain or partial-group products on the tensor
// cores, `bnd` channels to masked rank-2 updates. At most NVAR groups get a
// masked K copy; the full channels of further partial groups move to `bnd`,
// where their mask keeps every key (W_c >= dmax).
template <int D>
__device__ __forceinline__ void make_plan(const int32_t *cut, bool inter, int64_t N, int64_t qb, int64_t kb64,
                                          int lane, uint64_t &full, uint64_t &bnd) {
  constexpr int C = D / 2, G = D / 16;
  full = bnd = 0;
  int64_t dmin = 0, dmax = -1;
  if (!tile_distance_range(N, XBM, XSUB, qb, kb64, &dmin, &dmax)) return;  // the same in every lane
  const int k0 = classify_cutoff(dmin, dmax, cut[lane]);
  const int k1 = lane + 32 < C ? classify_cutoff(dmin, dmax, cut[lane + 32]) : TILE_SKIP;
  full = __ballot_sync(FULL, k0 == TILE_FULL) | (static_cast<uint64_t>(__ballot_sync(FULL, k1 == TILE_FULL)) << 32);
  bnd = __ballot_sync(FULL, k0 == TILE_BOUNDARY) |
        (static_cast<uint64_t>(__ballot_sync(FULL, k1 == TILE_BOUNDARY)) << 32);
  int nvar = 0;
  for (int g = 0; g < G; ++g) {
    const uint32_t keep = group_keep<D>(full, g, inter);
    if (keep == 0u || keep == 0xffffu) continue;
    if (++nvar <= NVAR) continue;
    // demoting removes every full channel of g, which can turn a group
    // counted before (half-split: g - D/32) from plain into partial, so the
    // count restarts; every restart removes a full channel, so it ends
    const uint64_t moved = full & group_chans<D>(g, inter);
    full &= ~moved;
    bnd |= moved;
    nvar = 0;
    g = -1;
  }
}

// Warp-wide: copy the 128-row Q group tile at `src` to `dst` (both 256-byte
// aligned, so the TMA 32-byte swizzle is the same), keeping the dims whose bit
// in `keep` is set and zeroing the rest; then fence the copy for the tensor
// core's async proxy. Row r's logical 16-byte chunk q sits at position
// q ^ ((r >> 2) & 1); lane l always moves chunks of logical index
// (l & 1) ^ ((l >> 3) & 1).
__device__ __forceinline__ void masked_q_copy(uint8_t *dst, const uint8_t *src, uint32_t keep, int lane) {
  const int q = (lane & 1) ^ ((lane >> 3) & 1);
  const uint32_t m8 = (keep >> (8 * q)) & 0xffu;
  uint32_t wm[4];
#pragma unroll
  for (int e = 0; e < 4; ++e)
    wm[e] = ((m8 >> (2 * e)) & 1u ? 0x0000ffffu : 0u) | ((m8 >> (2 * e + 1)) & 1u ? 0xffff0000u : 0u);
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int x = it * 32 + lane;  // 16-byte chunk index
    uint4 v = *reinterpret_cast<const uint4 *>(src + 16 * x);
    v.x &= wm[0];
    v.y &= wm[1];
    v.z &= wm[2];
    v.w &= wm[3];
    *reinterpret_cast<uint4 *>(dst + 16 * x) = v;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncwarp();
}

// Byte offset of (row, dim) in a 128-row x 16-dim bf16 tile stored with the
// TMA 32-byte swizzle (address bit 4 ^= bit 7).
__device__ __forceinline__ uint32_t sw32_offset(int row, int dim) {
  return 32u * row + 16u * (((dim >> 3) & 1) ^ ((row >> 2) & 1)) + 2u * (dim & 7);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Adds channel c's logits to this row's 64 S columns at the keys k >= cmin:
// S[k] += q_a k_a[k] + q_b k_b[k]. q_tile: the head's Q tile of group 0;
// k_tile: the K stage's group-0 tile advanced to the sub-tile's first key.
// Column chunks of 16 keys that every lane masks (k < cmin) or that lie
// past every lane's causal limit (k > kmax) are skipped.
template <int D>
__device__ __forceinline__ void add_channel(uint32_t (&su)[64], const uint8_t *q_tile, const uint8_t *k_tile, int r,
                                            int c, bool inter, int cmin, int kmax) {
  constexpr int C = D / 2;
  const int da = inter ? 2 * c : c, db = inter ? 2 * c + 1 : c + C;
  const int e = da & 15;
  const float qa = bf16_lo(*reinterpret_cast<const uint16_t *>(q_tile + (da >> 4) * XGROUP_BYTES + sw32_offset(r, e)));
  const float qb =
      bf16_lo(*reinterpret_cast<const uint16_t *>(q_tile + (db >> 4) * XGROUP_BYTES + sw32_offset(r, db & 15)));
  // key k of the sub-tile at 32k + (chunk position) + 2 (e & 7); the chunk
  // position flips with bit 2 of k
  const uint8_t *ka0 = k_tile + (da >> 4) * XGROUP_BYTES + 2 * (e & 7) + 16 * (e >> 3);
  const uint8_t *ka1 = k_tile + (da >> 4) * XGROUP_BYTES + 2 * (e & 7) + 16 * ((e >> 3) ^ 1);
  const uint32_t gap = static_cast<uint32_t>((db >> 4) - (da >> 4)) * XGROUP_BYTES;  // half-split: dim b's group
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (__all_sync(FULL, cmin >= 16 * j + 16 || kmax < 16 * j)) continue;
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      const int k = 16 * j + kk;
      const uint8_t *pa = ((k >> 2) & 1 ? ka1 : ka0) + 32 * k;
      float kav, kbv;
      if (inter) {
        const uint32_t w = *reinterpret_cast<const uint32_t *>(pa);
        kav = bf16_lo(w);
        kbv = bf16_hi(w);
      } else {
        kav = bf16_lo(*reinterpret_cast<const uint16_t *>(pa));
        kbv = bf16_lo(*reinterpret_cast<const uint16_t *>(pa + gap));
      }
      if (k >= cmin) su[k] = __float_as_uint(fmaf(qb, kbv, fmaf(qa, kav, __uint_as_float(su[k]))));
    }
  }
}

struct XBarriers {
  uint64_t *q_full, *k_full, *k_empty, *k_plan, *v_full, *v_empty, *s_ready, *p_ready, *o_ready, *o_final, *drain;
};

// PACKED: sequences located by cu_seqlens (else a uniform batch).
template <int D, bool PACKED>
__global__ void __launch_bounds__(XTHREADS, 1)
    prefill_exact_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ ChannelPrefillArgs a) {
  using L = XLayout<D>;
  constexpr int G = L::G, C = D / 2;
  constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, XSUB, false, false);
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, false, true);
  const bool inter = a.layout == WP_ROPE_INTERLEAVED;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::BAR_OFF);
  XBarriers B;
  B.q_full = bars;
  B.k_full = bars + 1;
  B.k_empty = B.k_full + XKST;
  B.k_plan = B.k_empty + XKST;  // the tile's plans are in the ring
  B.v_full = B.k_plan + XKST;
  B.v_empty = B.v_full + XVST;
  B.s_ready = B.v_empty + XVST;  // [2 heads][2 halves]
  B.p_ready = B.s_ready + 4;     // [2 heads][2 halves]
  B.o_ready = B.p_ready + 4;
  B.o_final = B.o_ready + 2;
  B.drain = B.o_final + 2;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::MISC_OFF);
  uint32_t *tmem_base_slot = reinterpret_cast<uint32_t *>(smem + L::MISC_OFF + 4);
  int32_t *cuts = reinterpret_cast<int32_t *>(smem + L::CUT_OFF);    // [plan][64]
  int32_t *gmax = reinterpret_cast<int32_t *>(smem + L::GMAX_OFF);   // [plan][8]
  uint64_t *ring = reinterpret_cast<uint64_t *>(smem + L::RING_OFF);  // [stage][plan][half][2]

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  // Grid (head pair within its KV group, query block, KV head x batch), as in
  // the grouped kernel.
  const int rep = a.Hq / a.Hkv;
  const int nslot = (rep % 2 == 0) ? 2 : 1;
  const int hk = static_cast<int>(blockIdx.z) % a.Hkv;
  const int b = static_cast<int>(blockIdx.z) / a.Hkv;
  const int h0 = hk * rep + static_cast<int>(blockIdx.x) * nslot;  // head of slot s = h0 + s
  const int nqb = (a.N + XBM - 1) / XBM;
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
    if (static_cast<int64_t>(qb) * XBM >= N) return;  // past this sequence's end (whole CTA)
  }
  // TMA row coordinate of query / key block x and the batch coordinate
  const auto block_row = [&](int x) { return PACKED ? static_cast<int>(row0 + static_cast<int64_t>(x) * XBM) : x * XBM; };
  const int bcoord = PACKED ? 0 : b;
  // one plan (cutoff row, masked copies) for both slots, or one per slot
  const int nplan = a.cut_rows == 1 ? 1 : nslot;
  const long long lim = a.wait_limit;

  if (threadIdx.x == 0) {
    *abort_flag = *reinterpret_cast<volatile int *>(&g_status) != 0 ? 1 : 0;
    mbar_init(B.q_full, 1);
    for (int s = 0; s < XKST; ++s) {
      mbar_init(&B.k_full[s], 1);
      mbar_init(&B.k_empty[s], 5 * nslot);  // per head: the MMA warp's commit and 4 softmax warps
      mbar_init(&B.k_plan[s], 1);
    }
    for (int s = 0; s < XVST; ++s) {
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
      mbar_init(&B.drain[s], 1);
    }
    fence_barrier_init();
  }
  for (int x = threadIdx.x; x < 2 * 64; x += XTHREADS) {
    const int p = x / 64, c = x % 64;
    cuts[x] = (c < C && p < nplan) ? a.cut[(a.cut_rows == 1 ? 0 : h0 + p) * C + c] : 0;
  }
  __syncthreads();
  if (threadIdx.x < 2 * 8) {
    const int p = threadIdx.x / 8, g = threadIdx.x % 8;
    int32_t m = -1;
    if (g < G && p < nplan)
      for (uint64_t cm = group_chans<D>(g, inter); cm; cm &= cm - 1) m = max(m, cuts[64 * p + __ffsll(cm) - 1]);
    gmax[threadIdx.x] = m;
  }
  if (warp == XMMA) {
    tmem_alloc(tmem_base_slot, XTMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_slot;
  const int nkb = *abort_flag ? 0 : qb + 1;  // key tiles qb, qb-1, ..., 0
  const int nsub = 2 * nkb;

  if (warp == XPRODUCER) {
    // ------------------------------------------------------------ producer
    // Q of both heads once; per key tile the K slices of the groups some
    // channel of either half (either plan) does not skip, then V one tile
    // behind. It never waits for a load to land, so two stay in flight.
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(B.q_full, nslot * G * XGROUP_BYTES);
      for (int s = 0; s < nslot; ++s)
        for (int g = 0; g < G; ++g)
          tma_load_4d(smem + L::Q_OFF + s * L::Q_SLOT + g * XGROUP_BYTES, &tm_q, B.q_full, 16 * g, h0 + s,
                      block_row(qb), bcoord);
    }
    __syncwarp();
    int k_issued = 0, v_issued = 0;
    bool ok = true;
    auto load_v = [&](int t) -> bool {
      const int st = t % XVST;
      if (t >= XVST && !warp_wait_idle(&B.v_empty[st], ((t / XVST) - 1) & 1, lim, abort_flag)) return false;
      if (leader) {
        mbar_arrive_expect_tx(&B.v_full[st], (D / 64) * XV_CHUNK);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(smem + L::V_OFF + st * L::V_STAGE + c * XV_CHUNK, &tm_v, &B.v_full[st], 64 * c, hk,
                      block_row(qb - t), bcoord);
      }
      __syncwarp();
      ++v_issued;
      return true;
    };
    for (int t = 0; ok && t < nkb; ++t) {
      const int st = t % XKST;
      if (t >= XKST && !warp_wait_idle(&B.k_empty[st], ((t / XKST) - 1) & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      uint32_t need = 0;
      for (int hh = 0; hh < 2; ++hh) {
        int64_t dmin, dmax;
        if (!tile_distance_range(N, XBM, XSUB, qb, 2 * (qb - t) + hh, &dmin, &dmax)) continue;
        for (int x = 0; x < 8 * nplan; ++x)
          if (static_cast<int64_t>(gmax[x]) >= dmin) need |= 1u << (x % 8);
      }
      need &= (1u << G) - 1u;
      if (leader) {
        mbar_arrive_expect_tx(&B.k_full[st], __popc(need) * XGROUP_BYTES);
        for (uint32_t m = need; m; m &= m - 1) {
          const int g = __ffs(m) - 1;
          tma_load_4d(smem + L::K_OFF + st * L::K_STAGE + g * XGROUP_BYTES, &tm_k, &B.k_full[st], 16 * g, hk,
                      block_row(qb - t), bcoord);
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
    for (int s = 0; s < XKST && s < k_issued; ++s) {
      const int last = s + ((k_issued - 1 - s) / XKST) * XKST;
      warp_wait_idle(&B.k_full[s], (last / XKST) & 1, lim, nullptr);
    }
    for (int s = 0; s < XVST && s < v_issued; ++s) {
      const int last = s + ((v_issued - 1 - s) / XVST) * XVST;
      warp_wait_idle(&B.v_full[s], (last / XVST) & 1, lim, nullptr);
    }
  } else if (warp == XFINISH) {
    // ------------------------------------------------------------ plan warp
    // Per key tile the channel plan of each (plan, half), once the tile two
    // back has released the ring entry (the stage's k_empty).
    for (int t = 0; t < nkb; ++t) {
      const int st = t % XKST;
      if (t >= XKST && !warp_wait_idle(&B.k_empty[st], ((t / XKST) - 1) & 1, lim, abort_flag)) break;
      uint64_t *rs = ring + st * 8;  // [plan][half][full, bnd]
      for (int p = 0; p < nplan; ++p)
        for (int hh = 0; hh < 2; ++hh) {
          uint64_t f, bd;
          make_plan<D>(cuts + 64 * p, inter, N, qb, 2 * (qb - t) + hh, lane, f, bd);
          if (lane == 0) {
            rs[4 * p + 2 * hh] = f;
            rs[4 * p + 2 * hh + 1] = bd;
          }
        }
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.k_plan[st]);
    }
  } else if (warp >= XMMA && warp < XMMA + nslot) {
    // ------------------------------------------------------- MMA issuers
    const int s = warp - XMMA;
    const int p = nplan == 1 ? 0 : s;
    const bool leader = elect_one();
    const uint64_t q_desc = smem_desc(smem_u32(smem + L::Q_OFF + s * L::Q_SLOT), 16, 256, SMEM_SWIZZLE_32B);
    const uint64_t k_desc = smem_desc(smem_u32(smem + L::K_OFF), 16, 256, SMEM_SWIZZLE_32B);
    uint8_t *qv = smem + L::QV_OFF + s * QSLOTS * XGROUP_BYTES;
    const uint64_t qv_desc = smem_desc(smem_u32(qv), 16, 256, SMEM_SWIZZLE_32B);
    const uint64_t v_desc = smem_desc(smem_u32(smem + L::V_OFF), XV_CHUNK, 1024, SMEM_SWIZZLE_128B);
    bool ok = warp_wait(B.q_full, 0, lim, abort_flag);
    constexpr uint32_t GD = XGROUP_BYTES >> 4;  // one group tile in descriptor units
    // The masked Q copies: slot j holds group (skey[j] >> 16) with kept dims
    // (skey[j] & 0xffff) and was last read by QK(suse[j]). QK(u) may
    // overwrite a slot unless QK(u - 1) reads it (QK(u - 2) and earlier have
    // completed: the softmax consumed their S before P(u - 2) freed the half
    // for u).
    uint32_t skey[QSLOTS];
    int suse[QSLOTS];
#pragma unroll
    for (int j = 0; j < QSLOTS; ++j) {
      skey[j] = 0xffffffffu;
      suse[j] = -4;
    }
    // copy slot of a partially kept group's key for QK(u), writing the copy
    // on a miss
    auto slot_for = [&](uint32_t key, int u) -> int {
      int found = -1;
#pragma unroll
      for (int j = 0; j < QSLOTS; ++j)
        if (skey[j] == key) found = j;
      if (found < 0) {
#pragma unroll
        for (int j = QSLOTS - 1; j >= 0; --j)
          if (suse[j] < u - 1) found = j;
        found = found < 0 ? 0 : found;  // never: at most NVAR slots are in use by QK(u - 1)
        masked_q_copy(qv + found * XGROUP_BYTES, smem + L::Q_OFF + s * L::Q_SLOT + (key >> 16) * XGROUP_BYTES,
                      key & 0xffffu, lane);
#pragma unroll
        for (int j = 0; j < QSLOTS; ++j)
          if (j == found) skey[j] = key;
      }
#pragma unroll
      for (int j = 0; j < QSLOTS; ++j)
        if (j == found) suse[j] = u;
      return found;
    };

    // QK of this head's sub-tile u into S half u & 1 (the tile's K and plans
    // are in): plain groups from Q, partially kept groups from masked copies.
    auto issue_qk = [&](int u) {
      const int t = u >> 1, hh = u & 1, st = t % XKST;
      const uint64_t full = ring[st * 8 + 4 * p + 2 * hh];
      const uint32_t s_col = tmem + xcol_s(s) + XSUB * hh;
      const uint64_t kst = k_desc + ((st * L::K_STAGE + hh * XHALF_BYTES) >> 4);
      // plain groups, and the partially kept ones (at most NVAR, as the
      // plan allows) with their kept dims: key = group << 16 | kept
      uint32_t plain = 0;
      uint32_t pkey0 = 0, pkey1 = 0;
      int npart = 0;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const uint32_t keep = group_keep<D>(full, g, inter);
        if (keep == 0xffffu) {
          plain |= 1u << g;
        } else if (keep != 0u && npart < NVAR) {
          const uint32_t key = (static_cast<uint32_t>(g) << 16) | keep;
          if (npart == 0) pkey0 = key;
          else pkey1 = key;
          ++npart;
        }
      }
      // descriptors of the partially kept groups' products, broadcast from
      // lane 0 so that they are warp-uniform values
      uint64_t pa0 = 0, pb0 = 0, pa1 = 0, pb1 = 0;
      if (npart > 0) {
        pa0 = qv_desc + slot_for(pkey0, u) * GD;
        pb0 = kst + (pkey0 >> 16) * GD;
      }
      if (npart > 1) {
        pa1 = qv_desc + slot_for(pkey1, u) * GD;
        pb1 = kst + (pkey1 >> 16) * GD;
      }
      if (npart > 0) {
        pa0 = __shfl_sync(FULL, pa0, 0);
        pb0 = __shfl_sync(FULL, pb0, 0);
        pa1 = __shfl_sync(FULL, pa1, 0);
        pb1 = __shfl_sync(FULL, pb1, 0);
      }
      if (leader) {
        // The plain groups first, with descriptors at fixed offsets from
        // loop-invariant bases (this issue loop is the MMA warp's hot path),
        // then the few partially kept ones from their copy slots.
        uint32_t acc = 0;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          if ((plain >> g) & 1u) {
            umma_ss(s_col, q_desc + g * GD, kst + g * GD, IDESC_QK, acc);
            acc = 1;
          }
        }
        if (npart > 0) {
          umma_ss(s_col, pa0, pb0, IDESC_QK, acc);
          acc = 1;
        }
        if (npart > 1) umma_ss(s_col, pa1, pb1, IDESC_QK, acc);
        umma_commit(&B.s_ready[2 * s + hh]);
      }
      __syncwarp();
    };
    // a key tile's K and plans
    auto tile_in = [&](int t) -> bool {
      const int st = t % XKST;
      if (!warp_wait(&B.k_full[st], (t / XKST) & 1, lim, abort_flag)) return false;
      if (!warp_wait(&B.k_plan[st], (t / XKST) & 1, lim, abort_flag)) return false;
      tc_fence_after();
      return true;
    };

    if (ok && nkb > 0) {
      ok = tile_in(0);
      if (ok) {
        issue_qk(0);
        issue_qk(1);
        if (leader) umma_commit(&B.k_empty[0]);
        __syncwarp();
      }
    }
    for (int u = 0; ok && u < nsub; ++u) {
      const int t = u >> 1, hh = u & 1;
      const int vst = t % XVST;
      if (hh == 0 && !warp_wait(&B.v_full[vst], (t / XVST) & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      const uint64_t vst_desc = v_desc + ((vst * L::V_STAGE) >> 4);
      if (!warp_wait(&B.p_ready[2 * s + hh], t & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t p_col = tmem + xcol_s(s) + XSUB * hh;
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < XSUB / 16; ++kk)
          umma_ts(tmem + xcol_o(s), p_col + kk * 8, vst_desc + (hh * (XSUB / 16) + kk) * (2048 >> 4), IDESC_PV,
                  (u > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&B.o_ready[s]);
        if (u == nsub - 1) umma_commit(&B.o_final[s]);
        if (hh == 1) umma_commit(&B.v_empty[vst]);
      }
      __syncwarp();
      if (u + 2 < nsub) {
        if (hh == 0 && !tile_in(t + 1)) {
          ok = false;
          break;
        }
        issue_qk(u + 2);
        if (hh == 1) {
          if (leader) umma_commit(&B.k_empty[(t + 1) % XKST]);
          __syncwarp();
        }
      }
    }
    if (leader) umma_commit(&B.drain[s]);
    __syncwarp();
    warp_wait(&B.drain[s], 0, lim, nullptr);
  } else if (warp / 4 < nslot) {
    // ------------------------------------------------------- softmax warps
    const int slot = warp / 4;
    const int q4 = warp % 4;
    const int p = nplan == 1 ? 0 : slot;
    const int r = q4 * 32 + lane;  // row of the query tile == TMEM lane
    const int h = h0 + slot;
    const int32_t *cut = cuts + 64 * p;
    const uint8_t *q_tile = smem + L::Q_OFF + slot * L::Q_SLOT;
    const int64_t i = static_cast<int64_t>(qb) * XBM + r;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const uint32_t o_addr = lane_addr + xcol_o(slot);
    const float c2 = a.scale_log2;
    const uint64_t c2x2 = pack_f2(c2, c2);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = nsub == 0 || warp_wait(B.q_full, 0, lim, abort_flag);
    uint64_t full1 = 0, bnd1 = 0;  // the plan of the tile's second half
    bool hold = false;             // this warp still reads the tile's K stage
    for (int u = 0; ok && u < nsub; ++u) {
      const int t = u >> 1, hh = u & 1, st = t % XKST;
      const int64_t k0 = static_cast<int64_t>(qb - t) * XBN + XSUB * hh;
      const uint32_t s_addr = lane_addr + xcol_s(slot) + XSUB * hh;
      uint64_t full, bnd;
      if (hh == 0) {
        // both halves' plans; without boundary work the tile's stage and ring
        // entry are released right away
        if (!warp_wait(&B.k_plan[st], (t / XKST) & 1, lim, abort_flag)) {
          ok = false;
          break;
        }
        full = ring[st * 8 + 4 * p];
        bnd = ring[st * 8 + 4 * p + 1];
        full1 = ring[st * 8 + 4 * p + 2];
        bnd1 = ring[st * 8 + 4 * p + 3];
        hold = (bnd | bnd1) != 0ull;
        if (!hold) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&B.k_empty[st]);
        } else if (!warp_wait(&B.k_full[st], (t / XKST) & 1, lim, abort_flag)) {  // K read below
          ok = false;
          break;
        }
      } else {
        full = full1;
        bnd = bnd1;
      }
      if (!warp_wait(&B.s_ready[2 * slot + hh], t & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t su[64];
      load_half(s_addr, full != 0ull, su);
      const uint8_t *k_tile = smem + L::K_OFF + st * L::K_STAGE + hh * XHALF_BYTES;
      const int kmax = t == 0 ? r - XSUB * hh : XSUB - 1;  // last causal key column of this row
      for (uint64_t m = bnd; m; m &= m - 1) {
        const int c = __ffsll(static_cast<long long>(m)) - 1;
        const int64_t cmin64 = i - k0 - cut[c];
        const int cmin = cmin64 < 0 ? 0 : (cmin64 > XSUB ? XSUB : static_cast<int>(cmin64));
        add_channel<D>(su, q_tile, k_tile, r, c, inter, cmin, kmax);
      }
      if (hh == 1 && hold) {  // this warp is done with tile t's K
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.k_empty[st]);
      }
      if (t == 0) causal_mask(su, XSUB * hh, r);
      const float m_half = half_max(su) * c2;
      if (u == 0) {
        m_run = m_half;
      } else if (__any_sync(FULL, m_half > m_run + RESCALE_THRESHOLD)) {
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
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      // a packed batch's diagonal tile takes every exponential on MUFU, so its
      // causally masked entries (possibly the next sequence's keys) give exactly 0
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
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.p_ready[2 * slot + hh]);
    }
    __nv_bfloat16 *orow = a.o + (((PACKED ? row0 : static_cast<int64_t>(b) * a.N) + i) * a.Hq + h) * D;
    float *lse_at = a.lse == nullptr ? nullptr
                                     : a.lse + (PACKED ? static_cast<int64_t>(h) * a.T + row0 + i
                                                       : (static_cast<int64_t>(b) * a.Hq + h) * a.N + i);
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
  if (warp == XMMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, XTMEM_COLS);
  }
}

template <int D>
cudaError_t launch_exact(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                         const ChannelPrefillArgs &a, cudaStream_t stream) {
  const int nqb = (a.N + XBM - 1) / XBM;
  const int rep = a.Hq / a.Hkv;
  const int nslot = rep % 2 == 0 ? 2 : 1;
  const uint32_t smem = XLayout<D>::BYTES;
  const dim3 grid(rep / nslot, nqb, a.Hkv * a.B);
  if (a.cu_seqlens != nullptr) {
    cudaError_t e = cudaFuncSetAttribute(prefill_exact_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    prefill_exact_kernel<D, true><<<grid, XTHREADS, smem, stream>>>(tq, tk, tv, a);
  } else {
    cudaError_t e = cudaFuncSetAttribute(prefill_exact_kernel<D, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    prefill_exact_kernel<D, false><<<grid, XTHREADS, smem, stream>>>(tq, tk, tv, a);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_exact(int d_h, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                 const ChannelPrefillArgs &a, cudaStream_t stream) {
  return d_h == 128 ? launch_exact<128>(tq, tk, tv, a, stream) : launch_exact<64>(tq, tk, tv, a, stream);
}

}  // namespace wp
