"""The prefill kernel's boundary procedure, replayed in numpy: the boundary
groups of a tile are accumulated one distinct cutoff at a time in ascending
order, the running logit tile is masked in place after each class (keep iff
i - j <= W), and the full groups are added on top unmasked. Because the
windows of ascending cutoffs are nested, this equals masking every group by
its own cutoff ([RN §2.3, Eq. (8)]: group g adds iff i - j <= W_g). Host only."""
import numpy as np
import pytest


def _kernel_order(P, W, dist, dmin, dmax):
    """P[g]: per-group partial products of one tile; W[g]: group cutoffs."""
    G = len(W)
    skip = [g for g in range(G) if dmin > W[g]]
    full = [g for g in range(G) if dmax <= W[g]]
    bnd = [g for g in range(G) if g not in skip and g not in full]
    S = np.zeros_like(P[0])
    for w in sorted(set(W[g] for g in bnd)):
        for g in bnd:
            if W[g] == w:
                S = S + P[g]
        S = np.where(dist <= w, S, 0.0)  # in place: the kernel zeroes columns with i - j > w
    for g in full:
        S = S + P[g]
    return S


@pytest.mark.parametrize("seed", range(6))
def test_in_place_class_masking_equals_per_group_masks(seed):
    rng = np.random.default_rng(seed)
    G, BM, BN = 8, 16, 12
    i0 = int(rng.integers(0, 300))
    j0 = int(rng.integers(0, max(1, i0 - 5)))
    i = i0 + np.arange(BM)[:, None]
    j = j0 + np.arange(BN)[None, :]
    dist = (i - j).astype(np.int64)
    causal = dist >= 0
    dmin, dmax = int(dist[causal].min()), int(dist[causal].max())
    # cutoffs on both sides of and inside the tile's range, with repeats
    W = [int(x) for x in rng.choice([dmin - 1, dmin, (dmin + dmax) // 2, dmax - 1, dmax, dmax + 7], size=G)]
    W = [max(w, 0) for w in W]
    P = rng.standard_normal((G, BM, BN))
    want = sum(np.where(dist <= W[g], P[g], 0.0) for g in range(G))
    got = _kernel_order(P, W, dist, dmin, dmax)
    np.testing.assert_allclose(got[causal], want[causal], rtol=1e-12, atol=1e-12)
