// Device helpers shared by the prefill kernels (grouped and exact per-channel):
// warp-uniform bounded waits, TMEM loads of S, the base-2 online softmax pieces
// (row max, exponentials on MUFU and on the FMA pipe, O rescale) and the
// ascending enumeration of boundary cutoffs. Inline device code only.
//
// The polynomial exp2 (POLY_PAIRS of every 8 exponent pairs): Cody-Waite
// reduction x = j + f, |f| <= 1/2, and a degree-3 minimax polynomial for 2^f
// (coefficients from a Remez fit, max relative error 7.5e-5, far below
// bf16's 2^-9 for P), scaled by 2^j in the exponent field, in packed f32x2
// arithmetic.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "wp_device.cuh"

namespace wp {
namespace {

constexpr uint32_t FULL = 0xffffffffu;

// Row-max growth (base-2 units) below which O is not rescaled.
constexpr float RESCALE_THRESHOLD = 8.0f;
#ifndef WP_POLY_PAIRS
#define WP_POLY_PAIRS 2
#endif
constexpr int POLY_PAIRS = WP_POLY_PAIRS;  // of every 8 exponent pairs, on the FMA pipe
static_assert(POLY_PAIRS >= 0 && POLY_PAIRS <= 8, "POLY_PAIRS counts pairs out of 8");

// Smallest cutoff among the boundary groups in `bnd` that is > prev
// (prev = -1 for the first); returns false when there is none. `mask` gets
// the groups sharing that cutoff.
__device__ __forceinline__ bool next_boundary_class(const int32_t *cut, uint32_t bnd, int64_t prev, int32_t *W,
                                                    uint32_t *mask) {
  int64_t best = INT64_MAX;
  for (uint32_t m = bnd; m; m &= m - 1) {
    const int64_t w = cut[__ffs(m) - 1];
    if (w > prev && w < best) best = w;
  }
  if (best == INT64_MAX) return false;
  uint32_t mk = 0;
  for (uint32_t m = bnd; m; m &= m - 1) {
    const int g = __ffs(m) - 1;
    if (static_cast<int64_t>(cut[g]) == best) mk |= 1u << g;
  }
  *W = static_cast<int32_t>(best);
  *mask = mk;
  return true;
}

// All lanes poll the barrier, then the warp agrees: the result is uniform and
// the warp is converged for the .sync.aligned TMEM instructions that follow.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, long long lim, volatile int *abort_flag) {
  const bool ok = mbar_wait(bar, parity, lim, abort_flag);
  return __all_sync(FULL, ok);
}

// The same wait for a warp off the critical path (the TMA producer, the plan
// warp): it polls and sleeps between polls, so that it takes no issue slots
// from the softmax warps sharing its SM sub-partition while it waits.
template <unsigned SLEEP_NS = 100>
__device__ __forceinline__ bool warp_wait_idle(uint64_t *bar, uint32_t parity, long long lim,
                                               volatile int *abort_flag) {
  bool ok = true;
  if (!mbar_test_wait(bar, parity)) {
    const long long t0 = clock64();
    while (!mbar_test_wait(bar, parity)) {
      if (abort_flag != nullptr && *abort_flag) {
        ok = false;
        break;
      }
      if (clock64() - t0 > lim) {
        record_status(WP_ERR_TIMEOUT);
        if (abort_flag != nullptr) *abort_flag = 1;
        ok = false;
        break;
      }
      __nanosleep(SLEEP_NS);
    }
  }
  return __all_sync(FULL, ok);
}

// 64 TMEM columns of this warp's lanes into r, with one wait for both loads;
// the registers pass through the wait so no use moves above it.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  tmem_ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
  tmem_ld32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31]), "+r"(r[32]), "+r"(r[33]), "+r"(r[34]), "+r"(r[35]),
                 "+r"(r[36]), "+r"(r[37]), "+r"(r[38]), "+r"(r[39]), "+r"(r[40]), "+r"(r[41]), "+r"(r[42]),
                 "+r"(r[43]), "+r"(r[44]), "+r"(r[45]), "+r"(r[46]), "+r"(r[47]), "+r"(r[48]), "+r"(r[49]),
                 "+r"(r[50]), "+r"(r[51]), "+r"(r[52]), "+r"(r[53]), "+r"(r[54]), "+r"(r[55]), "+r"(r[56]),
                 "+r"(r[57]), "+r"(r[58]), "+r"(r[59]), "+r"(r[60]), "+r"(r[61]), "+r"(r[62]), "+r"(r[63])
               :
               : "memory");
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ uint64_t pack_f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpack_f2(uint64_t v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ uint64_t fsub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x for a pair of exponents on the FMA pipe (see the file comment), in
// packed f32x2 arithmetic. x below -120 gives ~2^-120, which is 0 for every
// sum this kernel forms.
__device__ __forceinline__ void poly_exp2x2(uint64_t x2, float &p0, float &p1) {
  constexpr float C0 = 0.99992806f, C1 = 0.69326097f, C2 = 0.24261113f, C3 = 0.05517167f;
  constexpr float ROUND = 12582912.0f;  // 1.5 * 2^23: adding it rounds to an integer
  float x0, x1;
  unpack_f2(x2, x0, x1);
  x2 = pack_f2(fmaxf(x0, -120.f), fmaxf(x1, -120.f));
  const uint64_t t2 = fadd2(x2, pack_f2(ROUND, ROUND));   // low mantissa bits hold j = rint(x)
  const uint64_t f2 = fsub2(x2, fsub2(t2, pack_f2(ROUND, ROUND)));  // f = x - j in [-1/2, 1/2]
  uint64_t q2 = ffma2(pack_f2(C3, C3), f2, pack_f2(C2, C2));
  q2 = ffma2(q2, f2, pack_f2(C1, C1));
  q2 = ffma2(q2, f2, pack_f2(C0, C0));
  float t0, t1;
  unpack_f2(t2, t0, t1);
  unpack_f2(q2, p0, p1);
  // 2^j * 2^f: add j to the exponent field. The bits of t are those of ROUND
  // plus j, and ROUND's own bits vanish from a 23-bit left shift (unsigned:
  // the shift and the sum wrap modulo 2^32, which is the intent).
  p0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  p1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}

// 64 columns of S, or zeros when no product of the sub-tile was computed.
// Called after the S-ready barrier, when every MMA that used the half has
// completed: a sub-tile without products first writes zeros into its half,
// and every sub-tile then takes the same TMEM load. (Zeroing the registers
// on that path instead gives the 64 registers two definitions, and the
// merge costs register moves on every sub-tile.)
__device__ __forceinline__ void load_half(uint32_t taddr, bool any_group, uint32_t (&su)[64]) {
  if (!any_group) {
    uint32_t z[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) z[c] = 0u;
    tmem_st32(taddr, z);
    tmem_st32(taddr + 32, z);
    tmem_wait_st();
  }
  tmem_ld64(taddr, su);
}

// Causal mask of the diagonal tile: key column c0 + c comes after row r.
__device__ __forceinline__ void causal_mask(uint32_t (&su)[64], int c0, int r) {
#pragma unroll
  for (int c = 0; c < 64; ++c)
    if (c0 + c > r) su[c] = __float_as_uint(-INFINITY);
}

// Max of 64 values: 4 independent chains of 3-input max.
__device__ __forceinline__ float half_max(const uint32_t (&su)[64]) {
  float mx4[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float m = __uint_as_float(su[16 * j]);
#pragma unroll
    for (int k = 1; k < 15; k += 2) m = max3(m, __uint_as_float(su[16 * j + k]), __uint_as_float(su[16 * j + k + 1]));
    mx4[j] = fmaxf(m, __uint_as_float(su[16 * j + 15]));
  }
  return fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
}

// p = 2^(s*c2 - m) for 64 columns: one packed FMA per pair; POLY_PAIRS of 8
// pairs take the polynomial exp2, the rest the MUFU unit. Adds the p to the
// four packed partial sums and writes them as bf16 pairs (32 TMEM columns)
// to p_addr.
template <bool USE_POLY>
__device__ __forceinline__ void exp_half(const uint32_t (&su)[64], uint64_t c2x2, float m, uint64_t (&acc)[4],
                                         uint32_t p_addr) {
  const uint64_t negm = pack_f2(-m, -m);
  uint32_t pk[32];
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const uint64_t x2 = ffma2(pack_f2(__uint_as_float(su[2 * k]), __uint_as_float(su[2 * k + 1])), c2x2, negm);
    float x0, x1;
    unpack_f2(x2, x0, x1);
    float p0, p1;
    if (USE_POLY && (k & 7) >= 8 - POLY_PAIRS) {
      poly_exp2x2(x2, p0, p1);
    } else {
      p0 = fast_exp2(x0);
      p1 = fast_exp2(x1);
    }
    acc[k & 3] = fadd2(acc[k & 3], pack_f2(p0, p1));
    pk[k] = pack_bf16x2(p0, p1);
  }
  tmem_st32(p_addr, pk);
}

// Multiply n32 x 32 fp32 TMEM columns of this warp's lanes by alpha.
__device__ __forceinline__ void scale_cols_f32(uint32_t taddr, int n32, float alpha) {
#pragma unroll 1
  for (int c4 = 0; c4 < n32; ++c4) {
    uint32_t u[32];
    tmem_ld32(taddr + 32 * c4, u);
    tmem_wait_ld(u);
#pragma unroll
    for (int k = 0; k < 32; ++k) u[k] = __float_as_uint(__uint_as_float(u[k]) * alpha);
    tmem_st32(taddr + 32 * c4, u);
  }
  tmem_wait_st();
}

}  // namespace
}  // namespace wp
