// Tile classification shared by the host scheduler (wp_schedule) and the
// device kernels, so both mark every (query block, key block) the same way.
//
// WavePrune reading notes "WavePrune：RoPE 通常只需一个旋转周期", §2.3 (paper
// Sec. 3.3 and its three-row table): for a query block and a key block the
// pair distances form [l_D, r_D]; a group with cutoff d' is skipped when
// d' < l_D, computed without a mask when d' >= r_D, and masked otherwise.
// Author's thread "Guancheng Du @ducatiqwq", post (6/7), states the same rule.
#pragma once

#include <cstdint>

#if defined(__CUDACC__)
#define WP_HD __host__ __device__ __forceinline__
#else
#define WP_HD inline
#endif

namespace wp {

enum : int { TILE_SKIP = 0, TILE_FULL = 1, TILE_BOUNDARY = 2, TILE_NONE = 3 };

// Distance range [dmin, dmax] of the causal pairs (j <= i) of tile (qb, kb)
// over tokens 0..N-1 with BM x BN blocks. Returns false when the tile holds
// no causal pair. The largest distance pairs the tile's last query with its
// first key; the smallest is 0 when the query and key ranges overlap and
// first-query minus last-key otherwise.
WP_HD bool tile_distance_range(int64_t N, int BM, int BN, int64_t qb, int64_t kb, int64_t *dmin, int64_t *dmax) {
  const int64_t qs = qb * BM, ks = kb * BN;
  const int64_t qe = (qs + BM < N ? qs + BM : N) - 1;  // last query row
  const int64_t ke = (ks + BN < N ? ks + BN : N) - 1;  // last key
  if (qs > qe || ks > ke || ks > qe) return false;
  *dmax = qe - ks;
  *dmin = qs > ke ? qs - ke : 0;
  return true;
}

// Class of one cutoff W on a tile with causal distances [dmin, dmax].
WP_HD int classify_cutoff(int64_t dmin, int64_t dmax, int32_t W) {
  if (dmin > static_cast<int64_t>(W)) return TILE_SKIP;
  if (dmax <= static_cast<int64_t>(W)) return TILE_FULL;
  return TILE_BOUNDARY;
}

}  // namespace wp
