// WavePrune split-KV decode (HBM-bound) and the LSE combine.
//
// What it computes: the prefill definition's row len-1 (WavePrune reading
// notes "WavePrune：RoPE 通常只需一个旋转周期", §2.1 Eq. (6) with the grouped
// cutoffs of §2.3 Eq. (8)): for the query at position len-1 and key j at
// distance dist = len-1-j,
//   s_j = scale * sum_{g : dist <= W_g} q[16g:16g+16] . k_j[16g:16g+16],
// then softmax over j = 0..len-1 and O = sum_j p_j v_j. §2.3's table: in
// decode a skipped group's K need not be read at all — only V is read in full.
//
// Split kernel: one CTA per (split, KV head, sequence); the CTA's 4 warps each
// stream 16-key blocks of the split's key chunk through a private 3-stage
// shared-memory ring filled with 16-byte cp.async loads (coalesced along the
// head dim). A 16-byte K piece whose group is out of window for that key is
// copied with source size 0 (no bytes read, slot zero-filled), so the group
// adds exactly 0 to the logit. In the row layout [Lmax, d] the skipped K
// bytes only leave HBM untouched where a whole 128-byte line is out of
// window; finer holes are fetched with their line. In the group-major K layout
// [D/16, Lmax, 16] a group's keys are contiguous 32-byte records, so the keys
// a group skips form one contiguous range that is not read at all; there a
// warp loads one group of a 16-key block (512 contiguous bytes) per
// instruction. The GQA query heads of the
// KV head (H_q/H_kv <= 8) form the rows of warp-level bf16 mma.sync products
// (scores Q.K^T and P.V, fp32 accumulation); the online softmax keeps the row
// max and row sum with warp shuffles. The 4 warps merge their states in
// shared memory and write one partial (O normalised, LSE base 2) per split.
// Masked modes (the MASK template parameter): one group table per query head
// (the loads cover the union of the heads' windows; each head keeps a group's
// product per key only inside its own window), the exact per-channel rule of
// Eq. (6) (a channel's K dims zeroed per key before the product, the query
// having one position), and the exact rule with one channel table per query
// head (one product per query head on the K fragments masked by its row).
// Combine kernel: per (sequence, query head) merge the splits by LSE.
#include <cuda_bf16.h>
#include <cstdint>
#include <type_traits>

#include "wp_decode.h"
#include "wp_device.cuh"

namespace wp {

namespace {

constexpr int DEC_WARPS = 4;
constexpr int DEC_THREADS = DEC_WARPS * 32;
constexpr int KEYS = 16;   // keys per warp block
constexpr int STAGES = 3;  // cp.async ring depth per warp

template <int D>
struct DecLayout {
  static constexpr int PIECES = D / 8;                   // 16-byte pieces per row
  static constexpr uint32_t ROWB = D * 2;                // bytes per row
  static constexpr uint32_t TILE = KEYS * ROWB;          // one 16-key K (or V) block
  static constexpr uint32_t STAGE = 2 * TILE;            // K then V
  static constexpr uint32_t WARP_BYTES = STAGES * STAGE;
  static constexpr uint32_t RING_BYTES = DEC_WARPS * WARP_BYTES;
  // after the loop the ring is reused for the cross-warp merge
  static constexpr uint32_t MERGE_BYTES = DEC_WARPS * 8 * (D + 2) * 4;
  static constexpr uint32_t BYTES = RING_BYTES > MERGE_BYTES ? RING_BYTES : MERGE_BYTES;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + D, fp32.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte offset of 16-byte piece p of row r inside a block: pieces are XOR
// swizzled by the row so 8 rows read at one column hit 8 distinct banks.
template <int D>
__device__ __forceinline__ uint32_t piece_off(int r, int p) {
  return static_cast<uint32_t>(r) * DecLayout<D>::ROWB + static_cast<uint32_t>((p ^ (r & 7)) * 16);
}

struct NoDecodeTables {
  int32_t unused;
};
template <int MASK>
using DecodeTablesArg = typename std::conditional<MASK == DECODE_MASK_GROUP_SHARED, NoDecodeTables, DecodeTables>::type;

// Zeroes the bf16 halves of r (dims k and k+1 of one key) whose channel is out
// of window at distance dist: the exact per-channel rule on the K operand.
template <int D>
__device__ __forceinline__ uint32_t mask_channels(uint32_t r, int k, int64_t dist, const int32_t *ccut, int layout) {
  constexpr int C = D / 2;
  const int c0 = layout == WP_ROPE_INTERLEAVED ? k >> 1 : k % C;
  const int c1 = layout == WP_ROPE_INTERLEAVED ? k >> 1 : (k + 1) % C;
  const uint32_t keep = (dist <= ccut[c0] ? 0x0000ffffu : 0u) | (dist <= ccut[c1] ? 0xffff0000u : 0u);
  return r & keep;
}

template <int D, int R, bool KGM, bool PAGED, int MASK>
__global__ void __launch_bounds__(DEC_THREADS)
    decode_split_kernel(const DecodeArgs a, const __grid_constant__ DecodeTablesArg<MASK> tabs) {
  using L = DecLayout<D>;
  constexpr int PIECES = L::PIECES;
  constexpr int KSTEPS = D / 16;
  constexpr int NT = D / 8;  // output n-tiles of 8 dims
  extern __shared__ __align__(128) uint8_t dsmem[];

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int len = a.lens[b];
  if (len < 1 || len > a.Lmax) return;  // the combine writes NaN for this sequence
  const int start = split * a.chunk;
  const int end = min(start + a.chunk, len);
  const int hq0 = hk * R;
  const int64_t part = (static_cast<int64_t>(b) * a.Hq + hq0) * a.nsplit + split;  // head hq0's slot
  if (start >= len) {
    if (threadIdx.x < R) a.lse_part[part + static_cast<int64_t>(threadIdx.x) * a.nsplit] = -INFINITY;
    return;
  }
  if (PAGED) {
    // A block-table entry outside [0, n_pages) poisons this split (LSE +inf):
    // the combine then writes NaN rows for the sequence; nothing is read.
    bool bad = false;
    for (int j = start / a.page_size + lane; j <= (end - 1) / a.page_size; j += 32) {
      const int pg = a.block_table[static_cast<int64_t>(b) * a.max_pages + j];
      bad = bad || pg < 0 || pg >= a.n_pages;
    }
    if (__any_sync(0xffffffffu, bad)) {
      if (threadIdx.x < R) a.lse_part[part + static_cast<int64_t>(threadIdx.x) * a.nsplit] = INFINITY;
      return;
    }
  }
  const int g = lane >> 2, t = lane & 3;
  const int64_t qpos = len - 1;
  // masked modes: the R heads' group rows or the channel cutoffs in shared memory
  int32_t *mcut = reinterpret_cast<int32_t *>(dsmem + L::BYTES);
  if constexpr (MASK == DECODE_MASK_GROUP_PER_HEAD) {
    for (int e = threadIdx.x; e < R * 8; e += DEC_THREADS)
      mcut[e] = (e % 8) < D / 16 ? tabs.head_cut[(hq0 + e / 8) * (D / 16) + e % 8] : WP_CUTOFF_INF;
  } else if constexpr (MASK == DECODE_MASK_CHANNEL) {
    for (int e = threadIdx.x; e < D / 2; e += DEC_THREADS) mcut[e] = tabs.chan_cut[e];
  } else if constexpr (MASK == DECODE_MASK_CHANNEL_PER_HEAD) {
    // the channel rows of the KV head's R query heads, row r at mcut + r * D / 2
    for (int e = threadIdx.x; e < R * (D / 2); e += DEC_THREADS)
      mcut[e] = tabs.head_chan_cut[(hq0 + e / (D / 2)) * (D / 2) + e % (D / 2)];
  }
  if constexpr (MASK != DECODE_MASK_GROUP_SHARED) __syncthreads();
  // exact rule: the cutoffs of the channels that own this lane's B-fragment
  // dims (16c + 2t, +1, 16c + 8 + 2t, +1 of every k-step c), held in registers
  int32_t lcut[MASK == DECODE_MASK_CHANNEL ? KSTEPS : 1][4];
  if constexpr (MASK == DECODE_MASK_CHANNEL) {
#pragma unroll
    for (int c = 0; c < KSTEPS; ++c) {
      const int k0 = 16 * c + 2 * t, k1 = k0 + 8;
      lcut[c][0] = mcut[a.layout == WP_ROPE_INTERLEAVED ? k0 >> 1 : k0 % (D / 2)];
      lcut[c][1] = mcut[a.layout == WP_ROPE_INTERLEAVED ? k0 >> 1 : (k0 + 1) % (D / 2)];
      lcut[c][2] = mcut[a.layout == WP_ROPE_INTERLEAVED ? k1 >> 1 : k1 % (D / 2)];
      lcut[c][3] = mcut[a.layout == WP_ROPE_INTERLEAVED ? k1 >> 1 : (k1 + 1) % (D / 2)];
    }
  }

  // Q as the A operand (rows = query heads; rows >= R and 8..15 are zero).
  uint32_t qa[KSTEPS][2];
  {
    const __nv_bfloat16 *qrow = a.q + (static_cast<int64_t>(b) * a.Hq + hq0 + (g < R ? g : 0)) * D;
#pragma unroll
    for (int c = 0; c < KSTEPS; ++c) {
      uint32_t lo = 0, hi = 0;
      if (g < R) {
        lo = *reinterpret_cast<const uint32_t *>(qrow + 16 * c + 2 * t);
        hi = *reinterpret_cast<const uint32_t *>(qrow + 16 * c + 8 + 2 * t);
      }
      qa[c][0] = lo;
      qa[c][1] = hi;
    }
  }

  const __nv_bfloat16 *kbase = a.kc + (static_cast<int64_t>(b) * a.Hkv + hk) * a.Lmax * D;  // either layout
  const __nv_bfloat16 *vbase = a.vc + (static_cast<int64_t>(b) * a.Hkv + hk) * a.Lmax * D;
  // Where the 16 keys from kb0 on live: K (row of kb0, or group 0 of kb0 in
  // the group-major layout, groups kgs elements apart) and V (row of kb0). A
  // paged cache holds page_size keys per page; a 16-key block never crosses a
  // page (page_size is a multiple of 16).
  auto block_src = [&](int kb0, const __nv_bfloat16 *&kblk, const __nv_bfloat16 *&vblk, int64_t &kgs) {
    if (PAGED) {
      const int64_t page = a.block_table[static_cast<int64_t>(b) * a.max_pages + kb0 / a.page_size];
      const int off = kb0 % a.page_size;
      const int64_t pbase = (page * a.Hkv + hk) * a.page_size * D;  // both layouts: one page per (page, head)
      kblk = a.kc + pbase + (KGM ? static_cast<int64_t>(off) * 16 : static_cast<int64_t>(off) * D);
      vblk = a.vc + pbase + static_cast<int64_t>(off) * D;
      kgs = static_cast<int64_t>(a.page_size) * 16;
    } else if (KGM && a.k_windowed) {
      kblk = a.kc + (static_cast<int64_t>(b) * a.Hkv + hk) * a.wstride;  // the (b, hk) rings; per group below
      vblk = vbase + static_cast<int64_t>(kb0) * D;
      kgs = 0;
    } else {
      kblk = kbase + (KGM ? static_cast<int64_t>(kb0) * 16 : static_cast<int64_t>(kb0) * D);
      vblk = vbase + static_cast<int64_t>(kb0) * D;
      kgs = static_cast<int64_t>(a.Lmax) * 16;
    }
  };
  const uint32_t ring = smem_u32(dsmem) + warp * L::WARP_BYTES;
  // This warp's blocks: start + 16*(warp + 4n).
  const int first = start + KEYS * warp;
  const int stride = KEYS * DEC_WARPS;
  // Windowed rings: the slot of the next block to load in each group's ring,
  // advanced by stride mod capacity per block (the blocks load in order).
  int wslot[8], wstep[8];
#pragma unroll
  for (int gi = 0; gi < 8; ++gi) {
    const int cap = (KGM && !PAGED && a.k_windowed && gi < D / 16) ? a.wcap[gi] : 16;
    wslot[gi] = first % cap;
    wstep[gi] = stride % cap;
  }

  // Issue the loads of one 16-key block into stage `st` (blocks in order).
  auto load_block = [&](int kb0, int st) {
    const uint32_t kdst = ring + st * L::STAGE, vdst = kdst + L::TILE;
    const __nv_bfloat16 *kblk, *vblk;
    int64_t kgs;
    block_src(kb0, kblk, vblk, kgs);
#pragma unroll
    for (int it = 0; it < KEYS * PIECES / 32; ++it) {
      const int idx = it * 32 + lane;
      const int r = idx / PIECES, p = idx % PIECES;
      const int key = kb0 + r;
      const bool valid = key < end;
      const int64_t rr = valid ? r : 0;  // any in-range address when nothing is read
      if (!KGM) {
        const int64_t dist = qpos - key;
        const bool kin = valid && dist <= static_cast<int64_t>(a.cut[p >> 1]);
        // An out-of-window K piece is copied with source size 0: nothing is
        // read and its shared-memory slot is zero-filled, so the group adds
        // exactly 0 to the score.
        cp_async16(kdst + piece_off<D>(r, p), kblk + rr * D + 8 * p, kin ? 16u : 0u);
      }
      cp_async16(vdst + piece_off<D>(r, p), vblk + rr * D + 8 * p, valid ? 16u : 0u);
    }
    if (KGM) {
      // group-major K: iteration gi takes group gi, lane = 2 * key + half
#pragma unroll
      for (int gi = 0; gi < D / 16; ++gi) {
        const int r = lane >> 1, half = lane & 1;
        const int key = kb0 + r;
        const bool valid = key < end;
        const int64_t rr = valid ? r : 0;
        const bool kin = valid && qpos - key <= static_cast<int64_t>(a.cut[gi]);
        // windowed rings: kb0 is a multiple of 16 and so is every capacity,
        // so the block's 16 slots are contiguous in the ring
        const __nv_bfloat16 *src = (!PAGED && a.k_windowed)
                                       ? kblk + a.wbase[gi] + (static_cast<int64_t>(wslot[gi]) + rr) * 16
                                       : kblk + gi * kgs + rr * 16;
        cp_async16(kdst + piece_off<D>(r, 2 * gi + half), src + 8 * half, kin ? 16u : 0u);
      }
      if (!PAGED && a.k_windowed) {
#pragma unroll
        for (int gi = 0; gi < D / 16; ++gi) {
          wslot[gi] += wstep[gi];
          if (wslot[gi] >= a.wcap[gi]) wslot[gi] -= a.wcap[gi];
        }
      }
    }
  };

  float m_run = -INFINITY, l_run = 0.f;  // for query head g (rows g < R)
  float o[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;

  const int nblk = first < end ? (end - first + stride - 1) / stride : 0;
#pragma unroll
  for (int s = 0; s < STAGES - 1; ++s) {
    if (s < nblk) load_block(first + s * stride, s);
    cp_async_commit();
  }
  for (int n = 0; n < nblk; ++n) {
    if (n + STAGES - 1 < nblk) load_block(first + (n + STAGES - 1) * stride, (n + STAGES - 1) % STAGES);
    cp_async_commit();
    cp_async_wait<STAGES - 1>();
    __syncwarp();
    const int st = n % STAGES;
    const uint32_t ks = ring + st * L::STAGE, vs = ks + L::TILE;
    const int kb0 = first + n * stride;

    // scores S[head][key] for keys 0-7 (s0) and 8-15 (s1)
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < KSTEPS; ++c) {
      const int mi = lane >> 3, rr = (mi >> 1) * 8 + (lane & 7), pp = 2 * c + (mi & 1);
      uint32_t b00, b01, b10, b11;
      ldsm_x4(ks + piece_off<D>(rr, pp), b00, b01, b10, b11);
      if constexpr (MASK == DECODE_MASK_CHANNEL) {
        // b00/b01: key g, dims 16c + 2t (+1) and 16c + 8 + 2t (+1); b10/b11: key 8 + g.
        // Distances fit 32 bits (Lmax < 2^31).
        const int d0 = static_cast<int>(qpos - (kb0 + g)), d1 = d0 - 8;
        b00 &= (d0 <= lcut[c][0] ? 0x0000ffffu : 0u) | (d0 <= lcut[c][1] ? 0xffff0000u : 0u);
        b01 &= (d0 <= lcut[c][2] ? 0x0000ffffu : 0u) | (d0 <= lcut[c][3] ? 0xffff0000u : 0u);
        b10 &= (d1 <= lcut[c][0] ? 0x0000ffffu : 0u) | (d1 <= lcut[c][1] ? 0xffff0000u : 0u);
        b11 &= (d1 <= lcut[c][2] ? 0x0000ffffu : 0u) | (d1 <= lcut[c][3] ? 0xffff0000u : 0u);
      }
      if constexpr (MASK == DECODE_MASK_CHANNEL_PER_HEAD) {
        // one product per query head r, with the shared K fragments masked by
        // head r's channel row; lanes of row g keep head g's product
        const int64_t d0 = qpos - (kb0 + g), d1 = d0 - 8;
#pragma unroll 1
        for (int r = 0; r < R; ++r) {
          const int32_t *hc = mcut + r * (D / 2);
          const uint32_t m00 = mask_channels<D>(b00, 16 * c + 2 * t, d0, hc, a.layout);
          const uint32_t m01 = mask_channels<D>(b01, 16 * c + 8 + 2 * t, d0, hc, a.layout);
          const uint32_t m10 = mask_channels<D>(b10, 16 * c + 2 * t, d1, hc, a.layout);
          const uint32_t m11 = mask_channels<D>(b11, 16 * c + 8 + 2 * t, d1, hc, a.layout);
          float t0[4] = {0.f, 0.f, 0.f, 0.f}, t1[4] = {0.f, 0.f, 0.f, 0.f};
          mma_16816(t0, qa[c][0], 0u, qa[c][1], 0u, m00, m01);
          mma_16816(t1, qa[c][0], 0u, qa[c][1], 0u, m10, m11);
          if (g == r) {
            s0[0] += t0[0];
            s0[1] += t0[1];
            s1[0] += t1[0];
            s1[1] += t1[1];
          }
        }
      } else if constexpr (MASK == DECODE_MASK_GROUP_PER_HEAD) {
        // this group's products apart, then kept per head (row g) and key
        float t0[4] = {0.f, 0.f, 0.f, 0.f}, t1[4] = {0.f, 0.f, 0.f, 0.f};
        mma_16816(t0, qa[c][0], 0u, qa[c][1], 0u, b00, b01);
        mma_16816(t1, qa[c][0], 0u, qa[c][1], 0u, b10, b11);
        const int64_t W = mcut[(g < R ? g : 0) * 8 + c];
        const int64_t d0 = qpos - (kb0 + 2 * t), d2 = d0 - 8;
        s0[0] += d0 <= W ? t0[0] : 0.f;
        s0[1] += d0 - 1 <= W ? t0[1] : 0.f;
        s1[0] += d2 <= W ? t1[0] : 0.f;
        s1[1] += d2 - 1 <= W ? t1[1] : 0.f;
      } else {
        mma_16816(s0, qa[c][0], 0u, qa[c][1], 0u, b00, b01);
        mma_16816(s1, qa[c][0], 0u, qa[c][1], 0u, b10, b11);
      }
    }
    // lane holds head g, keys 2t, 2t+1 (s0[0..1]) and 8+2t, 9+2t (s1[0..1])
    float sc[4] = {s0[0], s0[1], s1[0], s1[1]};
    const int kk[4] = {2 * t, 2 * t + 1, 8 + 2 * t, 9 + 2 * t};
    float mx = -INFINITY;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      sc[e] = (kb0 + kk[e] < end) ? sc[e] * a.scale_log2 : -INFINITY;
      mx = fmaxf(mx, sc[e]);
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    const float alpha = fast_exp2(m_run - m_new);
    float p[4], ps = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      p[e] = fast_exp2(sc[e] - m_new);
      ps += p[e];
    }
    ps += __shfl_xor_sync(0xffffffffu, ps, 1);
    ps += __shfl_xor_sync(0xffffffffu, ps, 2);
    l_run = l_run * alpha + ps;
    m_run = m_new;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      o[j][0] *= alpha;
      o[j][1] *= alpha;
    }
    const uint32_t pa0 = pack_bf16x2(p[0], p[1]), pa2 = pack_bf16x2(p[2], p[3]);
#pragma unroll
    for (int c = 0; c < KSTEPS; ++c) {
      const int mi = lane >> 3, rr = (mi & 1) * 8 + (lane & 7), pp = 2 * c + (mi >> 1);
      uint32_t b0a, b1a, b0b, b1b;
      ldsm_x4_t(vs + piece_off<D>(rr, pp), b0a, b1a, b0b, b1b);
      mma_16816(o[2 * c], pa0, 0u, pa2, 0u, b0a, b1a);
      mma_16816(o[2 * c + 1], pa0, 0u, pa2, 0u, b0b, b1b);
    }
    __syncwarp();
  }
  cp_async_wait<0>();
  __syncthreads();

  // Merge the 4 warps: warp w's state for head g goes to shared memory.
  float *merge = reinterpret_cast<float *>(dsmem);
  float *mw = merge + warp * 8 * (D + 2);  // [8 heads][D + 2]: O..., m, l
  if (g < R) {
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      mw[g * (D + 2) + 8 * j + 2 * t] = o[j][0];
      mw[g * (D + 2) + 8 * j + 2 * t + 1] = o[j][1];
    }
    if (t == 0) {
      mw[g * (D + 2) + D] = m_run;
      mw[g * (D + 2) + D + 1] = l_run;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < R * D; e += DEC_THREADS) {
    const int h = e / D, d = e % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < DEC_WARPS; ++w) M = fmaxf(M, merge[w * 8 * (D + 2) + h * (D + 2) + D]);
    float Lsum = 0.f, acc = 0.f;
#pragma unroll
    for (int w = 0; w < DEC_WARPS; ++w) {
      const float *mh = merge + w * 8 * (D + 2) + h * (D + 2);
      const float f = mh[D] == -INFINITY ? 0.f : fast_exp2(mh[D] - M);
      Lsum += mh[D + 1] * f;
      acc += mh[d] * f;
    }
    const int64_t slot = part + static_cast<int64_t>(h) * a.nsplit;
    a.o_part[slot * D + d] = acc / Lsum;
    if (d == 0) a.lse_part[slot] = M + __log2f(Lsum);
  }
}

template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const DecodeArgs a) {
  const int bh = blockIdx.x;
  const int b = bh / a.Hq;
  const int d = threadIdx.x;
  const int len = a.lens[b];
  __nv_bfloat16 *orow = a.o + static_cast<int64_t>(bh) * D;
  if (len < 1 || len > a.Lmax) {
    orow[d] = __float2bfloat16_rn(__int_as_float(0x7fc00000));
    if (d == 0 && a.lse != nullptr) a.lse[bh] = __int_as_float(0x7fc00000);
    return;
  }
  const int ns = (len + a.chunk - 1) / a.chunk;  // splits that hold keys
  const float *lp = a.lse_part + static_cast<int64_t>(bh) * a.nsplit;
  const float *op = a.o_part + static_cast<int64_t>(bh) * a.nsplit * D;
  float M = -INFINITY;
  for (int s = 0; s < ns; ++s) M = fmaxf(M, lp[s]);
  float Lsum = 0.f, acc = 0.f;
  for (int s = 0; s < ns; ++s) {
    const float w = fast_exp2(lp[s] - M);
    Lsum += w;
    acc += w * op[static_cast<int64_t>(s) * D + d];
  }
  orow[d] = __float2bfloat16_rn(acc / Lsum);
  if (d == 0 && a.lse != nullptr) a.lse[bh] = (M + log2f(Lsum)) * 0.69314718055994531f;
}

template <int D, int R, bool KGM, bool PAGED, int MASK>
cudaError_t launch_split_l(const DecodeArgs &a, const DecodeTables *tables, cudaStream_t stream) {
  const uint32_t smem = DecLayout<D>::BYTES + (MASK == DECODE_MASK_GROUP_SHARED         ? 0u
                                               : MASK == DECODE_MASK_CHANNEL_PER_HEAD ? R * (D / 2) * 4u
                                                                                      : 256u);
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D, R, KGM, PAGED, MASK>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.nsplit, a.Hkv, a.B);
  DecodeTablesArg<MASK> tabs;
  if constexpr (MASK == DECODE_MASK_GROUP_SHARED)
    tabs.unused = 0;
  else
    tabs = *tables;
  decode_split_kernel<D, R, KGM, PAGED, MASK><<<grid, DEC_THREADS, smem, stream>>>(a, tabs);
  return cudaGetLastError();
}

template <int D, int R>
cudaError_t launch_split(const DecodeArgs &a, const DecodeTables *tables, cudaStream_t stream) {
  if (a.mask == DECODE_MASK_GROUP_PER_HEAD)  // contiguous caches only (checked on the host)
    return a.k_group_major ? launch_split_l<D, R, true, false, DECODE_MASK_GROUP_PER_HEAD>(a, tables, stream)
                           : launch_split_l<D, R, false, false, DECODE_MASK_GROUP_PER_HEAD>(a, tables, stream);
  if (a.mask == DECODE_MASK_CHANNEL)
    return a.k_group_major ? launch_split_l<D, R, true, false, DECODE_MASK_CHANNEL>(a, tables, stream)
                           : launch_split_l<D, R, false, false, DECODE_MASK_CHANNEL>(a, tables, stream);
  if (a.mask == DECODE_MASK_CHANNEL_PER_HEAD)
    return a.k_group_major ? launch_split_l<D, R, true, false, DECODE_MASK_CHANNEL_PER_HEAD>(a, tables, stream)
                           : launch_split_l<D, R, false, false, DECODE_MASK_CHANNEL_PER_HEAD>(a, tables, stream);
  if (a.block_table != nullptr)
    return a.k_group_major ? launch_split_l<D, R, true, true, 0>(a, tables, stream)
                           : launch_split_l<D, R, false, true, 0>(a, tables, stream);
  return a.k_group_major ? launch_split_l<D, R, true, false, 0>(a, tables, stream)
                         : launch_split_l<D, R, false, false, 0>(a, tables, stream);
}

// One thread per 16-byte piece of the group-major output, in output order:
// consecutive threads write consecutive bytes.
template <int D>
__global__ void kcache_group_major_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst, int64_t BH,
                                          int Lmax) {
  constexpr int G = D / 16;
  const int64_t n = BH * G * Lmax * 2;
  for (int64_t o = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; o < n;
       o += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int half = static_cast<int>(o & 1);
    const int64_t key = (o >> 1) % Lmax;
    const int64_t bg = (o >> 1) / Lmax;  // bh * G + g
    const int g = static_cast<int>(bg % G);
    const int64_t bh = bg / G;
    dst[o] = src[(bh * Lmax + key) * (D / 8) + 2 * g + half];
  }
}

template <int D>
cudaError_t launch_split_r(const DecodeArgs &a, const DecodeTables *tables, int R, cudaStream_t stream) {
  switch (R) {
    case 1: return launch_split<D, 1>(a, tables, stream);
    case 2: return launch_split<D, 2>(a, tables, stream);
    case 4: return launch_split<D, 4>(a, tables, stream);
    default: return launch_split<D, 8>(a, tables, stream);
  }
}

}  // namespace

// The windowed cache's ring geometry, by value into the kernels below.
struct WindowGeom {
  int32_t wcap[8];
  int64_t wbase[8];
  int64_t wstride;
};

// One thread per (b, hk, group, slot) 16-byte half: the latest key j < len
// with j % cap == slot, or zeros.
__global__ void kcache_window_from_rows_kernel(const uint4 *__restrict__ src, const int32_t *__restrict__ lens,
                                               uint4 *__restrict__ dst, int B, int Hkv, int Lmax, int D,
                                               const __grid_constant__ WindowGeom geo) {
  const int G = D / 16;
  const int64_t per_bh = geo.wstride / 8;  // uint4 per (b, hk)
  const int64_t total = static_cast<int64_t>(B) * Hkv * per_bh;
  for (int64_t x = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; x < total;
       x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t bh = x / per_bh, e = (x % per_bh) * 8;  // element offset within (b, hk)
    int g = G - 1;
    while (g > 0 && e < geo.wbase[g]) --g;
    const int64_t cap = geo.wcap[g];
    const int64_t within = e - geo.wbase[g];
    const int64_t slot = within / 16, half = (within % 16) / 8;
    const int len = lens[bh / Hkv];
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (len >= 1 && len <= Lmax && slot <= len - 1) {
      const int64_t j = slot + cap * ((len - 1 - slot) / cap);
      v = src[((bh * Lmax + j) * D + 16 * g) / 8 + half];
    }
    dst[x] = v;
  }
}

// One thread per (b, hk, group, half): the new key of sequence b into slot pos % cap.
__global__ void kcache_window_append_kernel(const uint4 *__restrict__ k_new, const int32_t *__restrict__ pos,
                                            uint4 *__restrict__ dst, int B, int Hkv, int Lmax, int D,
                                            const __grid_constant__ WindowGeom geo) {
  const int G = D / 16;
  const int64_t total = static_cast<int64_t>(B) * Hkv * G * 2;
  for (int64_t x = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; x < total;
       x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t bh = x / (G * 2);
    const int g = static_cast<int>((x / 2) % G), half = static_cast<int>(x % 2);
    const int p = pos[bh / Hkv];
    if (p < 0 || p >= Lmax) continue;  // outside the cache: nothing written
    const int64_t slot = p % geo.wcap[g];
    dst[(bh * geo.wstride + geo.wbase[g] + slot * 16) / 8 + half] = k_new[(bh * D + 16 * g) / 8 + half];
  }
}

cudaError_t launch_kcache_group_major(const __nv_bfloat16 *src, __nv_bfloat16 *dst, int64_t BH, int Lmax, int D,
                                      cudaStream_t stream) {
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const uint4 *s = reinterpret_cast<const uint4 *>(src);
  uint4 *d = reinterpret_cast<uint4 *>(dst);
  if (D == 128)
    kcache_group_major_kernel<128><<<nsm * 8, 256, 0, stream>>>(s, d, BH, Lmax);
  else
    kcache_group_major_kernel<64><<<nsm * 8, 256, 0, stream>>>(s, d, BH, Lmax);
  return cudaGetLastError();
}

static WindowGeom window_geom(const int32_t *wcap, const int64_t *wbase, int64_t wstride) {
  WindowGeom g;
  for (int k = 0; k < 8; ++k) {
    g.wcap[k] = wcap[k];
    g.wbase[k] = wbase[k];
  }
  g.wstride = wstride;
  return g;
}

cudaError_t launch_kcache_window_from_rows(const __nv_bfloat16 *src, const int32_t *lens, __nv_bfloat16 *dst, int B,
                                           int Hkv, int Lmax, int D, const int32_t *wcap, const int64_t *wbase,
                                           int64_t wstride, cudaStream_t stream) {
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  kcache_window_from_rows_kernel<<<nsm * 8, 256, 0, stream>>>(reinterpret_cast<const uint4 *>(src), lens,
                                                              reinterpret_cast<uint4 *>(dst), B, Hkv, Lmax, D,
                                                              window_geom(wcap, wbase, wstride));
  return cudaGetLastError();
}

cudaError_t launch_kcache_window_append(const __nv_bfloat16 *k_new, const int32_t *pos, __nv_bfloat16 *dst, int B,
                                        int Hkv, int Lmax, int D, const int32_t *wcap, const int64_t *wbase,
                                        int64_t wstride, cudaStream_t stream) {
  const int64_t total = static_cast<int64_t>(B) * Hkv * (D / 16) * 2;
  const int grid = static_cast<int>((total + 255) / 256 < 4096 ? (total + 255) / 256 : 4096);
  kcache_window_append_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4 *>(k_new), pos,
                                                        reinterpret_cast<uint4 *>(dst), B, Hkv, Lmax, D,
                                                        window_geom(wcap, wbase, wstride));
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs &a, const DecodeTables *tables, int d_h, cudaStream_t stream) {
  const int R = a.Hq / a.Hkv;
  cudaError_t e =
      d_h == 128 ? launch_split_r<128>(a, tables, R, stream) : launch_split_r<64>(a, tables, R, stream);
  if (e != cudaSuccess) return e;
  if (d_h == 128)
    decode_combine_kernel<128><<<a.B * a.Hq, 128, 0, stream>>>(a);
  else
    decode_combine_kernel<64><<<a.B * a.Hq, 64, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace wp
