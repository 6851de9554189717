// WavePrune grouped-cutoff causal prefill: backward pass (dQ, dK, dV).
//
// What it computes: the gradients of sum(dO * O) through the forward
// definition (WavePrune reading notes "WavePrune：RoPE 通常只需一个旋转周期",
// §2.1 Eq. (6), §2.3 Eq. (8)): with P_ij = exp(L_ij - LSE_i) from the
// forward's LSE and D_i = <dO_i, O_i>,
//   dV_j = sum_i P_ij dO_i,   dS_ij = P_ij (<dO_i, V_j> - D_i),
//   dQ_i[g] = scale * sum_j 1[i - j <= W_g] dS_ij K_j[g],
//   dK_j[g] = scale * sum_i 1[i - j <= W_g] dS_ij Q_i[g]   (16-dim group g).
// §2.3 (its paragraph on the backward kernel) states the two facts this
// follows: in the backward the head dimension is the output axis of the dQ
// and dK products, so the group mask is applied to the gradient operand dS
// before the product (one masked copy of dS per boundary group; full groups
// use dS as it is; skipped groups add nothing), and dQ and dK are formed
// from the same masked operands.
//
// Three kernels on warp-level tensor-core products (mma.sync m16n8k16, bf16
// operands, fp32 accumulation), operands staged in shared memory with 16-byte
// cp.async copies:
//   delta_kernel   D_i = <dO_i, O_i> per row (fp32).
//   dq_kernel      one CTA per (64-query block, query head), 4 warps of 16
//                  query rows; it walks the key blocks j <= i and forms
//                  S = Q K^T (group by group, boundary groups masked per
//                  element), P, dP = dO V^T, dS, then dQ += (dS masked) K.
//   dkdv_kernel    one CTA per (64-key block, KV head), 4 warps of 16 keys;
//                  it walks the query heads of the KV head and the 32-query
//                  blocks i >= j and forms S^T = K Q^T, P^T, dP^T = V dO^T,
//                  dS^T, then dV += P^T dO and dK += (dS^T masked) Q. The GQA
//                  query heads add into one accumulator: no atomics.
// The logits are recomputed in both product kernels (7 products per tile
// pair instead of 5) so that neither needs a cross-CTA reduction.
#include <cuda_bf16.h>
#include <cstdint>

#include "wp_backward.h"
#include "wp_device.cuh"
#include "wp_tile.h"

namespace wp {

namespace {

constexpr int BWD_THREADS = 128;  // 4 warps
constexpr float LOG2E = 1.4426950408889634f;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// C(16x8, fp32) += A(16x16 bf16, row) * B(16x8 bf16, col).
__device__ __forceinline__ void mma(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Shared-memory tiles of rows of D bf16, padded by 16 bytes so the 8 rows an
// ldmatrix reads fall in distinct banks.
template <int D>
struct Rows {
  static constexpr uint32_t STRIDE = D * 2 + 16;
  static __device__ __forceinline__ uint32_t at(uint32_t base, int row, int col) {
    return base + static_cast<uint32_t>(row) * STRIDE + static_cast<uint32_t>(col) * 2;
  }
};

// Copies `rows` rows of D bf16 (global row stride `gstride` elements, rows
// from `first`, those at or beyond `limit` zero-filled) into a padded tile.
template <int D>
__device__ __forceinline__ void load_rows(uint32_t dst, const __nv_bfloat16 *src, int64_t gstride, int first,
                                          int rows, int limit) {
  constexpr int PIECES = D / 8;
  for (int idx = threadIdx.x; idx < rows * PIECES; idx += BWD_THREADS) {
    const int r = idx / PIECES, p = idx % PIECES;
    const bool valid = first + r < limit;
    const __nv_bfloat16 *g = src + (valid ? static_cast<int64_t>(first + r) * gstride : 0) + 8 * p;
    cp_async16(Rows<D>::at(dst, r, 8 * p), g, valid ? 16u : 0u);
  }
}

// A-operand fragments (16 rows x 16 keys, bf16) of the 16 x (8 * NT) fp32
// tile x, keys 16kk .. 16kk+15 from its n-tiles 2kk and 2kk+1.
template <int NT>
__device__ __forceinline__ void to_a_frags(const float (&x)[NT][4], uint32_t (&a)[NT / 2][4]) {
#pragma unroll
  for (int kk = 0; kk < NT / 2; ++kk) {
    a[kk][0] = pack_bf16x2(x[2 * kk][0], x[2 * kk][1]);
    a[kk][1] = pack_bf16x2(x[2 * kk][2], x[2 * kk][3]);
    a[kk][2] = pack_bf16x2(x[2 * kk + 1][0], x[2 * kk + 1][1]);
    a[kk][3] = pack_bf16x2(x[2 * kk + 1][2], x[2 * kk + 1][3]);
  }
}

// Class of group cutoff W on a block of pairs whose distances span
// [dmin, dmax] (no causal pair: dmax < 0, the group is skipped).
__device__ __forceinline__ int block_class(int64_t dmin, int64_t dmax, int32_t W) {
  if (dmax < 0) return TILE_SKIP;
  return classify_cutoff(dmin, dmax, W);
}

// ------------------------------------------------------------------ delta

template <int D>
__global__ void __launch_bounds__(BWD_THREADS) delta_kernel(const BackwardArgs a) {
  // one warp per (b, i, h) row, rows in [B, N, Hq] order
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (BWD_THREADS / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int64_t rows = static_cast<int64_t>(a.B) * a.N * a.Hq;
  if (row >= rows) return;
  const __nv_bfloat16 *o = a.o + row * D, *g = a.dout + row * D;
  float acc = 0.f;
  for (int e = lane; e < D; e += 32) acc = fmaf(__bfloat162float(o[e]), __bfloat162float(g[e]), acc);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    const int64_t h = row % a.Hq, i = (row / a.Hq) % a.N, b = row / (static_cast<int64_t>(a.Hq) * a.N);
    a.delta[(b * a.Hq + h) * a.N + i] = acc;
  }
}

// --------------------------------------------------------------------- dQ

constexpr int DQ_BQ = 64;  // query rows per CTA (4 warps x 16)
constexpr int DQ_BK = 64;  // keys per step

template <int D>
struct DqSmem {
  static constexpr uint32_t TILE = DQ_BQ * Rows<D>::STRIDE;
  static constexpr uint32_t Q = 0, DO = TILE, K = 2 * TILE, V = 4 * TILE;  // K, V: two stages each
  static constexpr uint32_t CUT = 6 * TILE;                                   // 8 int32
  static constexpr uint32_t BYTES = CUT + 32;
};

template <int D>
__global__ void __launch_bounds__(BWD_THREADS) dq_kernel(const __grid_constant__ BackwardArgs a) {
  constexpr int G = D / 16;
  using S = DqSmem<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  int32_t *cut_s = reinterpret_cast<int32_t *>(smem + S::CUT);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, gq = lane >> 2, tq = lane & 3;
  const int nqb = (a.N + DQ_BQ - 1) / DQ_BQ;
  const int qb = nqb - 1 - static_cast<int>(blockIdx.x);  // heaviest blocks first
  const int h = blockIdx.y, b = blockIdx.z;
  const int hk = h / (a.Hq / a.Hkv);
  const int q0 = qb * DQ_BQ;
  if (threadIdx.x < G) cut_s[threadIdx.x] = a.cut[(a.cut_rows == 1 ? 0 : h) * G + threadIdx.x];

  const int64_t qstride = static_cast<int64_t>(a.Hq) * D, kstride = static_cast<int64_t>(a.Hkv) * D;
  const __nv_bfloat16 *qg = a.q + (static_cast<int64_t>(b) * a.N * a.Hq + h) * D;
  const __nv_bfloat16 *dog = a.dout + (static_cast<int64_t>(b) * a.N * a.Hq + h) * D;
  const __nv_bfloat16 *kg = a.k + (static_cast<int64_t>(b) * a.N * a.Hkv + hk) * D;
  const __nv_bfloat16 *vg = a.v + (static_cast<int64_t>(b) * a.N * a.Hkv + hk) * D;
  load_rows<D>(sbase + S::Q, qg, qstride, q0, DQ_BQ, a.N);
  load_rows<D>(sbase + S::DO, dog, qstride, q0, DQ_BQ, a.N);
  load_rows<D>(sbase + S::K, kg, kstride, 0, DQ_BK, a.N);
  load_rows<D>(sbase + S::V, vg, kstride, 0, DQ_BK, a.N);
  cp_async_commit();

  // this thread's two query rows
  const int r0 = warp * 16 + gq;
  const int64_t i0 = q0 + r0, i1 = i0 + 8;
  const float *lse_h = a.lse + (static_cast<int64_t>(b) * a.Hq + h) * a.N;
  const float *del_h = a.delta + (static_cast<int64_t>(b) * a.Hq + h) * a.N;
  const float l2_0 = i0 < a.N ? lse_h[i0] * LOG2E : 0.f, l2_1 = i1 < a.N ? lse_h[i1] * LOG2E : 0.f;
  const float d_0 = i0 < a.N ? del_h[i0] : 0.f, d_1 = i1 < a.N ? del_h[i1] : 0.f;
  // the warp's rows [wi0, wi1] (clipped to N)
  const int64_t wi0 = q0 + warp * 16, wi1 = min(static_cast<int64_t>(a.N) - 1, wi0 + 15);

  float dq[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) dq[n][0] = dq[n][1] = dq[n][2] = dq[n][3] = 0.f;

  const int nkb = (q0 + DQ_BQ - 1) / DQ_BK + 1;  // key blocks with a key <= the block's last row
  for (int kb = 0; kb < nkb; ++kb) {
    const int st = kb & 1;
    if (kb + 1 < nkb) {
      load_rows<D>(sbase + S::K + (st ^ 1) * S::TILE, kg, kstride, (kb + 1) * DQ_BK, DQ_BK, a.N);
      load_rows<D>(sbase + S::V + (st ^ 1) * S::TILE, vg, kstride, (kb + 1) * DQ_BK, DQ_BK, a.N);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t ks = sbase + S::K + st * S::TILE, vs = sbase + S::V + st * S::TILE;
    const int64_t k0 = static_cast<int64_t>(kb) * DQ_BK;
    const int64_t kj1 = min(static_cast<int64_t>(a.N) - 1, k0 + DQ_BK - 1);
    const int64_t dmax = wi1 - k0, dmin = max(static_cast<int64_t>(0), wi0 - kj1);
    if (wi0 < a.N && dmax >= 0) {
      // dP = dO V^T
      float dp[8][4];
#pragma unroll
      for (int n = 0; n < 8; ++n) dp[n][0] = dp[n][1] = dp[n][2] = dp[n][3] = 0.f;
#pragma unroll
      for (int kd = 0; kd < D / 16; ++kd) {
        uint32_t fa[4];
        ldsm_x4(Rows<D>::at(sbase + S::DO, warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1), 16 * kd + 8 * (lane >> 4)),
                fa);
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t fb[4];
          ldsm_x4(Rows<D>::at(vs, 16 * np + (lane & 7) + 8 * (lane >> 4), 16 * kd + 8 * ((lane >> 3) & 1)), fb);
          mma(dp[2 * np], fa, fb[0], fb[1]);
          mma(dp[2 * np + 1], fa, fb[2], fb[3]);
        }
      }
      // S = sum over non-skipped groups of Q_g K_g^T, boundary groups masked
      float s[8][4];
#pragma unroll
      for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const int32_t W = cut_s[g];
        const int cls = block_class(dmin, dmax, W);
        if (cls == TILE_SKIP) continue;
        uint32_t fa[4];
        ldsm_x4(Rows<D>::at(sbase + S::Q, warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1), 16 * g + 8 * (lane >> 4)),
                fa);
        float t[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n) t[n][0] = t[n][1] = t[n][2] = t[n][3] = 0.f;
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t fb[4];
          ldsm_x4(Rows<D>::at(ks, 16 * np + (lane & 7) + 8 * (lane >> 4), 16 * g + 8 * ((lane >> 3) & 1)), fb);
          mma(t[2 * np], fa, fb[0], fb[1]);
          mma(t[2 * np + 1], fa, fb[2], fb[3]);
        }
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int64_t i = (e < 2) ? i0 : i1, j = k0 + 8 * n + 2 * tq + (e & 1);
            s[n][e] += (cls == TILE_FULL || i - j <= W) ? t[n][e] : 0.f;
          }
      }
      // P = exp(S * scale - LSE) on the causal pairs; dS = P (dP - D)
#pragma unroll
      for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int64_t i = (e < 2) ? i0 : i1, j = k0 + 8 * n + 2 * tq + (e & 1);
          const float p = (j <= i && j < a.N && i < a.N) ? exp2f(s[n][e] * a.scale_log2 - (e < 2 ? l2_0 : l2_1)) : 0.f;
          s[n][e] = p * (dp[n][e] - (e < 2 ? d_0 : d_1));
        }
      // dQ += (dS masked by group) K_g
      uint32_t dsa[4][4];
      to_a_frags<8>(s, dsa);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const int32_t W = cut_s[g];
        const int cls = block_class(dmin, dmax, W);
        if (cls == TILE_SKIP) continue;
        uint32_t ma[4][4];
        if (cls == TILE_BOUNDARY) {
          float m[8][4];
#pragma unroll
          for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int64_t i = (e < 2) ? i0 : i1, j = k0 + 8 * n + 2 * tq + (e & 1);
              m[n][e] = i - j <= W ? s[n][e] : 0.f;
            }
          to_a_frags<8>(m, ma);
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t fb[4];
          ldsm_x4_t(Rows<D>::at(ks, 16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1), 16 * g + 8 * (lane >> 4)), fb);
          if (cls == TILE_BOUNDARY) {
            mma(dq[2 * g], ma[kk], fb[0], fb[1]);
            mma(dq[2 * g + 1], ma[kk], fb[2], fb[3]);
          } else {
            mma(dq[2 * g], dsa[kk], fb[0], fb[1]);
            mma(dq[2 * g + 1], dsa[kk], fb[2], fb[3]);
          }
        }
      }
    }
    __syncthreads();  // the stage is reloaded two steps on
  }
  cp_async_wait<0>();
  // store dQ * scale
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    const int col = 8 * n + 2 * tq;
    if (i0 < a.N)
      *reinterpret_cast<uint32_t *>(a.dq + ((static_cast<int64_t>(b) * a.N + i0) * a.Hq + h) * D + col) =
          pack_bf16x2(dq[n][0] * a.scale, dq[n][1] * a.scale);
    if (i1 < a.N)
      *reinterpret_cast<uint32_t *>(a.dq + ((static_cast<int64_t>(b) * a.N + i1) * a.Hq + h) * D + col) =
          pack_bf16x2(dq[n][2] * a.scale, dq[n][3] * a.scale);
  }
}

// ---------------------------------------------------------------- dK, dV

constexpr int KV_BK = 64;  // keys per CTA (4 warps x 16)
constexpr int KV_BQ = 32;  // queries per step

template <int D>
struct KvSmem {
  static constexpr uint32_t KTILE = KV_BK * Rows<D>::STRIDE, QTILE = KV_BQ * Rows<D>::STRIDE;
  static constexpr uint32_t K = 0, V = KTILE, Q = 2 * KTILE, DO = Q + 2 * QTILE;  // Q, dO: two stages
  static constexpr uint32_t VEC = DO + 2 * QTILE;  // per stage: LSE*log2(e) [32], D [32]
  static constexpr uint32_t CUT = VEC + 2 * 2 * KV_BQ * 4;  // [rep][8] int32
  static uint32_t bytes(int rep) { return CUT + 32u * rep; }
};

template <int D>
__global__ void __launch_bounds__(BWD_THREADS) dkdv_kernel(const __grid_constant__ BackwardArgs a) {
  constexpr int G = D / 16;
  using S = KvSmem<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  float *vec = reinterpret_cast<float *>(smem + S::VEC);
  int32_t *cut_s = reinterpret_cast<int32_t *>(smem + S::CUT);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, gq = lane >> 2, tq = lane & 3;
  const int kb = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int rep = a.Hq / a.Hkv;
  const int kstart = kb * KV_BK;
  for (int e = threadIdx.x; e < rep * 8; e += BWD_THREADS) {
    const int r = e / 8, g = e % 8;
    cut_s[e] = g < G ? a.cut[(a.cut_rows == 1 ? 0 : hk * rep + r) * G + g] : WP_CUTOFF_INF;
  }

  const int64_t qstride = static_cast<int64_t>(a.Hq) * D, kstride = static_cast<int64_t>(a.Hkv) * D;
  const __nv_bfloat16 *kg = a.k + (static_cast<int64_t>(b) * a.N * a.Hkv + hk) * D;
  const __nv_bfloat16 *vg = a.v + (static_cast<int64_t>(b) * a.N * a.Hkv + hk) * D;
  load_rows<D>(sbase + S::K, kg, kstride, kstart, KV_BK, a.N);
  load_rows<D>(sbase + S::V, vg, kstride, kstart, KV_BK, a.N);

  // this thread's two keys
  const int64_t j0 = kstart + warp * 16 + gq, j1 = j0 + 8;
  const int64_t wj0 = kstart + warp * 16, wj1 = min(static_cast<int64_t>(a.N) - 1, wj0 + 15);

  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    dk[n][0] = dk[n][1] = dk[n][2] = dk[n][3] = 0.f;
    dv[n][0] = dv[n][1] = dv[n][2] = dv[n][3] = 0.f;
  }

  // steps: (query head r of the KV head, 32-query block from the key block's
  // first key on)
  const int qfirst = kstart / KV_BQ, nqblk = (a.N + KV_BQ - 1) / KV_BQ - qfirst;
  const int nsteps = rep * nqblk;
  auto load_step = [&](int step, int stg) {
    const int r = step / nqblk, qblk = qfirst + step % nqblk;
    const int h = hk * rep + r;
    const __nv_bfloat16 *qg = a.q + (static_cast<int64_t>(b) * a.N * a.Hq + h) * D;
    const __nv_bfloat16 *dog = a.dout + (static_cast<int64_t>(b) * a.N * a.Hq + h) * D;
    load_rows<D>(sbase + S::Q + stg * S::QTILE, qg, qstride, qblk * KV_BQ, KV_BQ, a.N);
    load_rows<D>(sbase + S::DO + stg * S::QTILE, dog, qstride, qblk * KV_BQ, KV_BQ, a.N);
    if (threadIdx.x < KV_BQ) {
      const int64_t i = static_cast<int64_t>(qblk) * KV_BQ + threadIdx.x;
      const int64_t off = (static_cast<int64_t>(b) * a.Hq + h) * a.N + i;
      vec[stg * 2 * KV_BQ + threadIdx.x] = i < a.N ? a.lse[off] * LOG2E : 0.f;
      vec[stg * 2 * KV_BQ + KV_BQ + threadIdx.x] = i < a.N ? a.delta[off] : 0.f;
    }
  };
  if (nsteps > 0) load_step(0, 0);
  cp_async_commit();

  for (int step = 0; step < nsteps; ++step) {
    const int stg = step & 1;
    if (step + 1 < nsteps) {
      __syncthreads();  // stage stg ^ 1 (and its vectors) are free: step - 1 is done
      load_step(step + 1, stg ^ 1);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const int r = step / nqblk;
    const int64_t i0blk = static_cast<int64_t>(qfirst + step % nqblk) * KV_BQ;
    const int64_t qi1 = min(static_cast<int64_t>(a.N) - 1, i0blk + KV_BQ - 1);
    const int64_t dmax = qi1 - wj0, dmin = max(static_cast<int64_t>(0), i0blk - wj1);
    if (wj0 >= a.N || dmax < 0) continue;  // no causal pair for this warp's keys
    const uint32_t qs = sbase + S::Q + stg * S::QTILE, dos = sbase + S::DO + stg * S::QTILE;
    const float *l2 = vec + stg * 2 * KV_BQ, *dl = l2 + KV_BQ;
    const int32_t *cut = cut_s + 8 * r;

    // dP^T = V dO^T (16 keys x 32 queries)
    float dpt[4][4];
#pragma unroll
    for (int n = 0; n < 4; ++n) dpt[n][0] = dpt[n][1] = dpt[n][2] = dpt[n][3] = 0.f;
#pragma unroll
    for (int kd = 0; kd < D / 16; ++kd) {
      uint32_t fa[4];
      ldsm_x4(Rows<D>::at(sbase + S::V, warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1), 16 * kd + 8 * (lane >> 4)),
              fa);
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        uint32_t fb[4];
        ldsm_x4(Rows<D>::at(dos, 16 * np + (lane & 7) + 8 * (lane >> 4), 16 * kd + 8 * ((lane >> 3) & 1)), fb);
        mma(dpt[2 * np], fa, fb[0], fb[1]);
        mma(dpt[2 * np + 1], fa, fb[2], fb[3]);
      }
    }
    // S^T = sum over non-skipped groups of K_g Q_g^T, boundary groups masked
    float st[4][4];
#pragma unroll
    for (int n = 0; n < 4; ++n) st[n][0] = st[n][1] = st[n][2] = st[n][3] = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int32_t W = cut[g];
      const int cls = block_class(dmin, dmax, W);
      if (cls == TILE_SKIP) continue;
      uint32_t fa[4];
      ldsm_x4(Rows<D>::at(sbase + S::K, warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1), 16 * g + 8 * (lane >> 4)),
              fa);
      float t[4][4];
#pragma unroll
      for (int n = 0; n < 4; ++n) t[n][0] = t[n][1] = t[n][2] = t[n][3] = 0.f;
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        uint32_t fb[4];
        ldsm_x4(Rows<D>::at(qs, 16 * np + (lane & 7) + 8 * (lane >> 4), 16 * g + 8 * ((lane >> 3) & 1)), fb);
        mma(t[2 * np], fa, fb[0], fb[1]);
        mma(t[2 * np + 1], fa, fb[2], fb[3]);
      }
#pragma unroll
      for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int64_t j = (e < 2) ? j0 : j1, i = i0blk + 8 * n + 2 * tq + (e & 1);
          st[n][e] += (cls == TILE_FULL || i - j <= W) ? t[n][e] : 0.f;
        }
    }
    // P^T on the causal pairs, then dS^T = P^T (dP^T - D)
    float pt[4][4];
#pragma unroll
    for (int n = 0; n < 4; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int64_t j = (e < 2) ? j0 : j1;
        const int c = 8 * n + 2 * tq + (e & 1);
        const int64_t i = i0blk + c;
        const float p = (j <= i && i < a.N && j < a.N) ? exp2f(st[n][e] * a.scale_log2 - l2[c]) : 0.f;
        pt[n][e] = p;
        st[n][e] = p * (dpt[n][e] - dl[c]);
      }
    // dV += P^T dO
    uint32_t pa[2][4];
    to_a_frags<4>(pt, pa);
#pragma unroll
    for (int kk = 0; kk < 2; ++kk)
#pragma unroll
      for (int nd = 0; nd < D / 16; ++nd) {
        uint32_t fb[4];
        ldsm_x4_t(Rows<D>::at(dos, 16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1), 16 * nd + 8 * (lane >> 4)), fb);
        mma(dv[2 * nd], pa[kk], fb[0], fb[1]);
        mma(dv[2 * nd + 1], pa[kk], fb[2], fb[3]);
      }
    // dK += (dS^T masked by group) Q_g
    uint32_t dsa[2][4];
    to_a_frags<4>(st, dsa);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int32_t W = cut[g];
      const int cls = block_class(dmin, dmax, W);
      if (cls == TILE_SKIP) continue;
      uint32_t ma[2][4];
      if (cls == TILE_BOUNDARY) {
        float m[4][4];
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int64_t j = (e < 2) ? j0 : j1, i = i0blk + 8 * n + 2 * tq + (e & 1);
            m[n][e] = i - j <= W ? st[n][e] : 0.f;
          }
        to_a_frags<4>(m, ma);
      }
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        uint32_t fb[4];
        ldsm_x4_t(Rows<D>::at(qs, 16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1), 16 * g + 8 * (lane >> 4)), fb);
        if (cls == TILE_BOUNDARY) {
          mma(dk[2 * g], ma[kk], fb[0], fb[1]);
          mma(dk[2 * g + 1], ma[kk], fb[2], fb[3]);
        } else {
          mma(dk[2 * g], dsa[kk], fb[0], fb[1]);
          mma(dk[2 * g + 1], dsa[kk], fb[2], fb[3]);
        }
      }
    }
  }
  cp_async_wait<0>();
  // store dK * scale and dV
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    const int col = 8 * n + 2 * tq;
    if (j0 < a.N) {
      const int64_t off = ((static_cast<int64_t>(b) * a.N + j0) * a.Hkv + hk) * D + col;
      *reinterpret_cast<uint32_t *>(a.dk + off) = pack_bf16x2(dk[n][0] * a.scale, dk[n][1] * a.scale);
      *reinterpret_cast<uint32_t *>(a.dv + off) = pack_bf16x2(dv[n][0], dv[n][1]);
    }
    if (j1 < a.N) {
      const int64_t off = ((static_cast<int64_t>(b) * a.N + j1) * a.Hkv + hk) * D + col;
      *reinterpret_cast<uint32_t *>(a.dk + off) = pack_bf16x2(dk[n][2] * a.scale, dk[n][3] * a.scale);
      *reinterpret_cast<uint32_t *>(a.dv + off) = pack_bf16x2(dv[n][2], dv[n][3]);
    }
  }
}

template <int D>
cudaError_t launch(const BackwardArgs &a, const BackwardMaps &maps, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(a.B) * a.N * a.Hq;
  delta_kernel<D><<<static_cast<unsigned>((rows + 3) / 4), BWD_THREADS, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_backward_dq_tc(D, a, maps, stream);
  if (e != cudaSuccess) return e;
  return launch_backward_dkdv_tc(D, a, maps, stream);
}

}  // namespace

cudaError_t launch_backward(int d_h, const BackwardArgs &a, const BackwardMaps &maps, cudaStream_t stream) {
  return d_h == 128 ? launch<128>(a, maps, stream) : launch<64>(a, maps, stream);
}

}  // namespace wp
