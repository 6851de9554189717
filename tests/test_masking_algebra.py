"""Two procedures of the prefill kernel, replayed in numpy (host only).

Boundary classes: the boundary groups of a tile are accumulated one distinct
cutoff at a time in ascending order, the running logit tile is masked in place
after each class (keep iff i - j <= W), and the full groups are added on top
unmasked. Because the windows of ascending cutoffs are nested, this equals
masking every group by its own cutoff ([RN §2.3, Eq. (8)]: group g adds iff
i - j <= W_g).

Online softmax with a stale running max: the max is raised (and O and the row
sum rescaled) only when a sub-tile's max exceeds it by more than 2^8 in base
2; in exact arithmetic the result is the softmax of the whole row."""
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


def _stale_max_softmax(s_tiles, v_tiles, c2, threshold=8.0):
    """The kernel's online softmax for one row, in fp64: base-2 exponents
    x = s*c2 - m with a running max m that is raised (rescaling O and the
    sum) only when a sub-tile's max exceeds it by more than `threshold`."""
    m = None
    o = np.zeros(v_tiles[0].shape[1])
    l = 0.0
    for s, v in zip(s_tiles, v_tiles):
        mt = s.max() * c2
        if m is None:
            m = mt
        elif mt > m + threshold:
            alpha = 2.0 ** (m - mt)
            o *= alpha
            l *= alpha
            m = mt
        p = 2.0 ** (s * c2 - m)
        o += p @ v
        l += p.sum()
    return o / l, m + np.log2(l)


@pytest.mark.parametrize("seed", range(5))
def test_stale_max_online_softmax_is_exact(seed):
    rng = np.random.default_rng(100 + seed)
    c2 = np.log2(np.e) / np.sqrt(128.0)
    tiles = 9
    # logits drift upward so the max grows, sometimes by more than 2^8 per tile
    s_tiles = [rng.standard_normal(64) * 20 + 40.0 * k * rng.random() for k in range(tiles)]
    v_tiles = [rng.standard_normal((64, 16)) for _ in range(tiles)]
    o, lse2 = _stale_max_softmax(s_tiles, v_tiles, c2)
    s = np.concatenate(s_tiles)
    v = np.concatenate(v_tiles)
    w = np.exp(s / np.sqrt(128.0) - (s / np.sqrt(128.0)).max())
    want = (w @ v) / w.sum()
    np.testing.assert_allclose(o, want, rtol=1e-10, atol=1e-12)
    want_lse = np.log(w.sum()) + (s / np.sqrt(128.0)).max()
    assert abs(lse2 * np.log(2.0) - want_lse) < 1e-9 * max(1.0, abs(want_lse))
