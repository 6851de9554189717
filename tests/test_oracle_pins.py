"""Pins for the fp64 oracle: checks against values and facts that do not come
from the oracle itself (printed worked values, closed forms, independent
library routines, brute force on tiny inputs).

Page tags:
  [RN] "WavePrune：RoPE 通常只需一个旋转周期" (reading notes of arXiv:2610.06963)
  [KC] "WavePrune：RoPE只用一个旋转周期，长文本性能反而更好"
  [TW] "Guancheng Du @ducatiqwq" (author's thread)
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "table12_qwen3_group_end_wavelengths.txt")


def _golden_rows():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            th, d, c, w = line.split()
            rows.append((float(th), int(d), int(c), int(w)))
    return rows


# --------------------------------------------------------------------------
# Cutoffs
# --------------------------------------------------------------------------

def test_table12_channel_cutoffs():
    """[RN §4.7, Table 12 and §2.1 teaching example]: printed wavelengths."""
    for theta, d, c, w in _golden_rows():
        wc, _ = oracle.cutoffs(d, theta, oracle.INTERLEAVED)
        assert wc[c] == w, (c, wc[c], w)


def test_table12_interleaved_group_cutoffs():
    """[RN §2.3 Eq. (8)] with 8 channels per group: group g's cutoff is that of
    its last channel 8g+7, which Table 12 prints for g = 0..5."""
    _, wg = oracle.cutoffs(128, 1e6, oracle.INTERLEAVED)
    assert list(wg[:6]) == [28, 160, 900, 5063, 28472, 160114]


def test_half_split_group_cutoffs_from_table12():
    """Half-split: dims [16g, 16g+16) belong to channels (16g mod 64) .. +15, so
    the group cutoff is that of channel 16(g mod 4)+15; Table 12 prints the
    values of channels 15, 31 and 47."""
    _, wg = oracle.cutoffs(128, 1e6, oracle.HALF_SPLIT)
    assert list(wg[:3]) == [160, 5063, 160114]
    assert list(wg[4:7]) == [160, 5063, 160114]
    assert wg[3] == wg[7]


@pytest.mark.parametrize("d,theta,scale", [(64, 1e4, 1.0), (128, 1e6, 1.0), (128, 1e6, 0.25)])
def test_cutoff_is_floor_of_one_period(d, theta, scale):
    """[RN §2.1]: keep iff distance <= floor(w_c), w_c = 2*pi/f_c, so
    W_c*f_c <= 2*pi < (W_c+1)*f_c. f_c recomputed here with math.pow. Also
    checks no w_c sits within 1e-6 of an integer, so the floor is stable."""
    wc, _ = oracle.cutoffs(d, theta, oracle.INTERLEAVED, scale_all=scale)
    for c in range(d // 2):
        f = scale * math.pow(theta, -2.0 * c / d)
        assert wc[c] * f <= 2 * math.pi < (wc[c] + 1) * f
        w = 2 * math.pi / f
        assert abs(w - round(w)) > 1e-6
    # cutoffs rise with the channel index [RN §1.1: larger c, lower frequency]
    assert np.all(np.diff(wc) >= 0)


def test_scaled_frequencies_move_cutoffs():
    """[RN §1.1]: with frequency scaling the cutoffs are recomputed from the
    scaled frequencies. Dividing every f_c by 4 equals keeping f_c and taking
    alpha = 8 (alpha*pi/(f/4) = 4*alpha*pi/f)."""
    a, ga = oracle.cutoffs(128, 1e6, oracle.HALF_SPLIT, scale_all=0.25)
    b, gb = oracle.cutoffs(128, 1e6, oracle.HALF_SPLIT, alpha=8.0)
    assert np.array_equal(a, b) and np.array_equal(ga, gb)
    # per-channel scale array behaves like the uniform one
    c, gc = oracle.cutoffs(128, 1e6, oracle.HALF_SPLIT, freq_scale=np.full(64, 0.25))
    assert np.array_equal(a, c) and np.array_equal(ga, gc)


def test_alpha_to_infinity_disables_pruning():
    """[RN §2.1]: alpha -> infinity means no pruning (cutoffs saturate)."""
    wc, wg = oracle.cutoffs(64, 1e4, oracle.INTERLEAVED, alpha=1e300)
    assert np.all(wc == np.iinfo(np.int32).max) and np.all(wg == np.iinfo(np.int32).max)


# --------------------------------------------------------------------------
# RoPE
# --------------------------------------------------------------------------

def _rope_complex(x, theta, layout, pos, scale_all=1.0):
    """Independent rotation: channel pairs as complex numbers times e^{i p f}."""
    B, N, H, d = x.shape
    C = d // 2
    f = scale_all * theta ** (-2.0 * np.arange(C) / d)
    ang = pos.reshape(B, N, 1, 1) * f.reshape(1, 1, 1, C)
    if layout == oracle.INTERLEAVED:
        z = x[..., 0::2] + 1j * x[..., 1::2]
    else:
        z = x[..., :C] + 1j * x[..., C:]
    z = z * np.exp(1j * ang)
    y = np.empty_like(x)
    if layout == oracle.INTERLEAVED:
        y[..., 0::2], y[..., 1::2] = z.real, z.imag
    else:
        y[..., :C], y[..., C:] = z.real, z.imag
    return y


@pytest.mark.parametrize("layout", [oracle.INTERLEAVED, oracle.HALF_SPLIT])
def test_rope_matches_complex_rotation(layout):
    """[KC RoPE matrix]: [[cos, -sin], [sin, cos]] on each pair at angle m*f."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal((2, 37, 3, 64))
    pos = rng.integers(0, 200000, size=(2, 37))
    y = oracle.rope(x, 1e4, layout, pos=pos)
    ref = _rope_complex(x, 1e4, layout, pos.astype(np.float64))
    assert np.max(np.abs(y - ref)) < 1e-9


def test_rope_half_split_matches_rotate_half():
    """Half-split reading: out = x*cos + rotate_half(x)*sin, the convention of
    the Qwen/Llama models the pages evaluate, written with torch ops."""
    g = torch.Generator().manual_seed(3)
    x = torch.randn(1, 20, 2, 128, generator=g, dtype=torch.float64)
    C = 64
    f = 1e6 ** (-2.0 * torch.arange(C, dtype=torch.float64) / 128)
    ang = torch.arange(20, dtype=torch.float64)[:, None] * f[None, :]
    cos = torch.cat([ang.cos(), ang.cos()], -1)[None, :, None, :]
    sin = torch.cat([ang.sin(), ang.sin()], -1)[None, :, None, :]
    rot = torch.cat([-x[..., C:], x[..., :C]], -1)
    ref = x * cos + rot * sin
    y = oracle.rope(x.numpy(), 1e6, oracle.HALF_SPLIT)
    assert np.max(np.abs(y - ref.numpy())) < 1e-12


@pytest.mark.parametrize("layout", [oracle.INTERLEAVED, oracle.HALF_SPLIT])
def test_rope_relative_position(layout):
    """[RN §1.1; abstract]: absolute positions cancel in q.k, leaving the
    relative position: <R(p)x, R(q)y> = <R(p-q)x, y>; norms are preserved."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal((1, 1, 1, 64))
    y = rng.standard_normal((1, 1, 1, 64))
    for p, q in [(5, 3), (1000, 17), (70000, 69999)]:
        a = oracle.rope(x, 1e4, layout, pos0=p).ravel() @ oracle.rope(y, 1e4, layout, pos0=q).ravel()
        b = oracle.rope(x, 1e4, layout, pos0=p - q).ravel() @ y.ravel()
        assert abs(a - b) < 1e-9
    r = oracle.rope(x, 1e4, layout, pos0=12345)
    assert abs(np.linalg.norm(r) - np.linalg.norm(x)) < 1e-12


def test_round_bf16_nearest_even():
    """The oracle's fp64 -> bf16 rounding returns the nearest bf16 and breaks
    exact ties to the even significand."""
    rng = np.random.default_rng(4)
    x = rng.standard_normal(20000) * np.exp(rng.uniform(-8, 8, 20000))
    bits = oracle.round_bf16_bits(x)
    r = oracle.bf16_bits_to_f64(bits)
    up = oracle.bf16_bits_to_f64((bits.astype(np.int32) + 1).astype(np.uint16))
    dn = oracle.bf16_bits_to_f64((bits.astype(np.int32) - 1).astype(np.uint16))
    err = np.abs(x - r)
    assert np.all(err <= np.abs(x - up)) and np.all(err <= np.abs(x - dn))
    # exact midpoints: 1 + 2^-8 lies between 1 (even) and 1 + 2^-7 (odd)
    mid = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8)])
    got = oracle.bf16_bits_to_f64(oracle.round_bf16_bits(mid))
    assert list(got) == [1.0, 1.0 + 2.0 ** -6, -1.0]


# --------------------------------------------------------------------------
# Logits and attention
# --------------------------------------------------------------------------

@pytest.mark.parametrize("mode", [oracle.MODE_CHANNEL, oracle.MODE_GROUPED])
@pytest.mark.parametrize("layout", [oracle.INTERLEAVED, oracle.HALF_SPLIT])
def test_single_channel_closed_form(mode, layout):
    """(c) [RN §1.1; TW (2/7)]: constant Q/K with one nonzero channel c give
    sqrt(d_h)*L_ij = m_Q m_K cos((i-j) f_c + omega) inside the window and 0
    outside. In grouped mode the window is the group's cutoff."""
    d, theta = 64, 1e4
    wc, wg = oracle.cutoffs(d, theta, layout)
    for c in [3, 5]:
        a, b = (2 * c, 2 * c + 1) if layout == oracle.INTERLEAVED else (c, c + d // 2)
        W = wc[c] if mode == oracle.MODE_CHANNEL else wg[a // 16]
        assert mode == oracle.MODE_CHANNEL or wg[a // 16] == wg[b // 16]
        N = int(W) + 12
        q = np.zeros(d)
        k = np.zeros(d)
        q[a], q[b] = 0.7, -1.3
        k[a], k[b] = -0.4, 0.9
        Q = oracle.rope(np.tile(q, (1, N, 1, 1)), theta, layout)[0, :, 0]
        K = oracle.rope(np.tile(k, (1, N, 1, 1)), theta, layout)[0, :, 0]
        cut = wc if mode == oracle.MODE_CHANNEL else wg
        L = oracle.logits(Q, K, cut, mode, layout)
        f = theta ** (-2.0 * c / d)
        omega = math.atan2(q[b], q[a]) - math.atan2(k[b], k[a])
        mq, mk = math.hypot(q[a], q[b]), math.hypot(k[a], k[b])
        for i in range(N):
            for j in range(i + 1):
                want = mq * mk * math.cos((i - j) * f + omega) if i - j <= W else 0.0
                assert abs(math.sqrt(d) * L[i, j] - want) < 1e-9, (i, j)
            assert np.all(np.isneginf(L[i, i + 1:]))


def _sdpa_reference(q, k, v):
    """Plain causal RoPE attention from torch library routines (fp64): SDPA
    with causal masking, GQA by repeating KV heads, LSE from logsumexp."""
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)  # B,H,N,d
    rep = q.shape[2] // k.shape[2]
    kt = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(rep, dim=1)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(rep, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    s = (qt @ kt.transpose(-1, -2)) / math.sqrt(q.shape[-1])
    N = q.shape[1]
    s = s.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), float("-inf"))
    return o.permute(0, 2, 1, 3).numpy(), torch.logsumexp(s, -1).numpy()


@pytest.mark.parametrize("mode", [oracle.MODE_GROUPED, oracle.MODE_CHANNEL])
def test_all_cutoffs_beyond_n_is_plain_rope_attention(mode):
    """(a) [RN §2.1]: alpha -> infinity (every cutoff >= N) is plain causal
    RoPE attention; compared with torch's SDPA on the same rotated inputs."""
    rng = np.random.default_rng(5)
    B, N, Hq, Hkv, d = 2, 48, 4, 2, 64
    q = oracle.rope(rng.standard_normal((B, N, Hq, d)), 1e4, oracle.HALF_SPLIT)
    k = oracle.rope(rng.standard_normal((B, N, Hkv, d)), 1e4, oracle.HALF_SPLIT)
    v = rng.standard_normal((B, N, Hkv, d))
    cut = np.full(d // 2 if mode == oracle.MODE_CHANNEL else d // 16, N)
    o, lse = oracle.attention(q, k, v, cut, mode, oracle.HALF_SPLIT)
    ro, rl = _sdpa_reference(q, k, v)
    assert np.max(np.abs(o - ro)) < 1e-12
    assert np.max(np.abs(lse - rl)) < 1e-12


def test_shift_invariance():
    """(b) [RN §1.1; abstract]: shifting every position by a constant leaves
    logits, and so outputs, unchanged (the mask depends on i-j only)."""
    rng = np.random.default_rng(6)
    N, d = 64, 64
    x_q = rng.standard_normal((1, N, 2, d))
    x_k = rng.standard_normal((1, N, 1, d))
    v = rng.standard_normal((1, N, 1, d))
    _, wg = oracle.cutoffs(d, 1e4, oracle.INTERLEAVED)
    outs = []
    for p0 in [0, 12345]:
        q = oracle.rope(x_q, 1e4, oracle.INTERLEAVED, pos0=p0)
        k = oracle.rope(x_k, 1e4, oracle.INTERLEAVED, pos0=p0)
        outs.append(oracle.attention(q, k, v, wg, oracle.MODE_GROUPED, oracle.INTERLEAVED))
    assert np.max(np.abs(outs[0][0] - outs[1][0])) < 1e-10
    assert np.max(np.abs(outs[0][1] - outs[1][1])) < 1e-10


@pytest.mark.parametrize("layout", [oracle.INTERLEAVED, oracle.HALF_SPLIT])
def test_channel_and_grouped_modes_agree_on_group_constant_cutoffs(layout):
    """(d) Eq. (6) vs Eq. (8) [RN §2.1, §2.3]: when every channel of a group
    has the same cutoff, the group max equals each channel's cutoff and the
    two definitions coincide."""
    rng = np.random.default_rng(7)
    d, N = 128, 96
    G, C = d // 16, d // 2
    levels = [3, 17, 40, 200]
    if layout == oracle.INTERLEAVED:
        wc = np.array([levels[(c // 8) % 4] for c in range(C)], dtype=np.int32)
        wg = np.array([levels[g % 4] for g in range(G)], dtype=np.int32)
    else:
        wc = np.array([levels[c // 16] for c in range(C)], dtype=np.int32)
        wg = np.array([levels[g % 4] for g in range(G)], dtype=np.int32)
    q = rng.standard_normal((1, N, 2, d))
    k = rng.standard_normal((1, N, 1, d))
    v = rng.standard_normal((1, N, 1, d))
    a = oracle.attention(q, k, v, wc, oracle.MODE_CHANNEL, layout)
    b = oracle.attention(q, k, v, wg, oracle.MODE_GROUPED, layout)
    assert np.max(np.abs(a[0] - b[0])) < 1e-12 and np.max(np.abs(a[1] - b[1])) < 1e-12
    # and they differ once the cutoffs inside a group differ
    wc2 = wc.copy()
    wc2[0] = 0
    c = oracle.attention(q, k, v, wc2, oracle.MODE_CHANNEL, layout)
    assert np.max(np.abs(c[0] - a[0])) > 1e-6


@pytest.mark.parametrize("mode", [oracle.MODE_GROUPED, oracle.MODE_CHANNEL])
def test_all_cutoffs_zero_closed_form(mode):
    """(f) [RN §2.1, detail 1]: a dropped term is 0, not -inf. With every
    cutoff 0 only the diagonal logit survives: L_ii = scale*q_i.k_i and every
    other causal logit is exactly 0, so
      O_i = (e^{s_ii} v_i + sum_{j<i} v_j) / (e^{s_ii} + i),
      LSE_i = ln(e^{s_ii} + i)."""
    rng = np.random.default_rng(8)
    N, d = 40, 64
    q = rng.standard_normal((1, N, 1, d))
    k = rng.standard_normal((1, N, 1, d))
    v = rng.standard_normal((1, N, 1, d))
    cut = np.zeros(d // 2 if mode == oracle.MODE_CHANNEL else d // 16, dtype=np.int32)
    o, lse = oracle.attention(q, k, v, cut, mode, oracle.INTERLEAVED)
    s = np.einsum("nd,nd->n", q[0, :, 0], k[0, :, 0]) / math.sqrt(d)
    csum = np.cumsum(v[0, :, 0], axis=0)
    for i in range(N):
        prev = csum[i - 1] if i > 0 else 0.0
        want = (math.exp(s[i]) * v[0, i, 0] + prev) / (math.exp(s[i]) + i)
        assert np.max(np.abs(o[0, i, 0] - want)) < 1e-12
        assert abs(lse[0, 0, i] - math.log(math.exp(s[i]) + i)) < 1e-12


def test_boundary_distance_is_inclusive():
    """[RN §2.1]: the keep rule uses <= at the first-period boundary: a pair at
    distance exactly W keeps the group, at W+1 it does not."""
    d = 64
    q = np.zeros((3, d))
    k = np.zeros((3, d))
    q[:, :16] = 1.0
    k[:, :16] = 1.0
    cut = np.array([1, 0, 0, 0], dtype=np.int32)
    L = oracle.logits(q, k, cut, oracle.MODE_GROUPED, oracle.INTERLEAVED, scale=1.0)
    assert L[1, 0] == 16.0   # distance 1 == W: kept
    assert L[2, 0] == 0.0    # distance 2 > W: dropped, logit 0 (not -inf)


def test_decode_equals_last_prefill_row():
    """(g) Decode at length L is prefill row L-1 over the same keys."""
    rng = np.random.default_rng(9)
    B, Hq, Hkv, d, Lmax = 3, 4, 2, 64, 70
    lens = np.array([70, 1, 33], dtype=np.int32)
    kc = rng.standard_normal((B, Hkv, Lmax, d))
    vc = rng.standard_normal((B, Hkv, Lmax, d))
    q = rng.standard_normal((B, Hq, d))
    _, wg = oracle.cutoffs(d, 1e4, oracle.INTERLEAVED)
    wg = np.minimum(wg, 20)
    o, lse = oracle.decode(q, kc, vc, lens, wg)
    for b in range(B):
        L = int(lens[b])
        k = kc[b].transpose(1, 0, 2)[None, :L]
        v = vc[b].transpose(1, 0, 2)[None, :L]
        rows = (np.zeros(Hq), np.arange(Hq), np.full(Hq, L - 1))
        ro, rl = oracle.attention_rows(q[b], rows, k, v, Hq, wg)
        assert np.max(np.abs(o[b] - ro)) < 1e-13 and np.max(np.abs(lse[b] - rl)) < 1e-13


# --------------------------------------------------------------------------
# Tile classes
# --------------------------------------------------------------------------

def _closed_form_counts(nqb, Bk, W):
    """Square blocks, N = nqb*Bk: a tile at block offset delta = qb - kb >= 1
    spans distances [(delta-1)Bk+1, (delta+1)Bk-1]; the diagonal spans
    [0, Bk-1]; there are nqb - delta tiles at offset delta."""
    skip = full = bnd = 0
    for delta in range(nqb):
        lo = 0 if delta == 0 else (delta - 1) * Bk + 1
        hi = (delta + 1) * Bk - 1 if delta else Bk - 1
        n = nqb - delta
        if W < lo:
            skip += n
        elif W >= hi:
            full += n
        else:
            bnd += n
    return skip, full, bnd


@pytest.mark.parametrize("W", [0, 5, 127, 128, 160, 300, 5063, 10 ** 6])
def test_tile_counts_closed_form(W):
    """(e) [RN §2.3 table; TW (6/7)]: skip if d' < l_D, full if d' >= r_D."""
    for nqb, Bk in [(8, 64), (5, 128)]:
        _, counts = oracle.tile_classes(nqb * Bk, Bk, Bk, [W], want_map=False)
        assert tuple(counts[0]) == _closed_form_counts(nqb, Bk, W)


@pytest.mark.parametrize("N,BM,BN", [(300, 128, 128), (257, 64, 128), (200, 128, 64), (1, 128, 128)])
def test_tile_classes_ragged_vs_numpy(N, BM, BN):
    """Ragged N and unequal blocks: the oracle's pair loop against a
    vectorised numpy distance matrix per tile."""
    cut = np.array([0, 3, 60, 130, 250, 10 ** 6], dtype=np.int32)
    cls, counts = oracle.tile_classes(N, BM, BN, cut)
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    dist = np.where(j <= i, i - j, -1)
    want_counts = np.zeros((cut.size, 3), dtype=np.int64)
    for qb in range(cls.shape[0]):
        for kb in range(cls.shape[1]):
            blk = dist[qb * BM:(qb + 1) * BM, kb * BN:(kb + 1) * BN]
            valid = blk[blk >= 0]
            for g, w in enumerate(cut):
                if valid.size == 0:
                    want = 3
                elif w < valid.min():
                    want = 0
                elif w >= valid.max():
                    want = 1
                else:
                    want = 2
                assert cls[qb, kb, g] == want
                if want < 3:
                    want_counts[g, want] += 1
    assert np.array_equal(counts, want_counts)


def test_paired_order_is_the_half_split_model_in_channel_mode():
    """Moving channel c's half-split pair (c, c + d/2) to dims (2c, 2c+1) of
    both Q and K leaves the exact per-channel rule unchanged ([RN §2.1, Eq.
    (6)] depends on channels, not on where their dims sit): the interleaved
    layout on the permuted data gives the half-split result on the original."""
    rng = np.random.default_rng(5)
    B, N, Hq, Hkv, d = 1, 40, 2, 1, 32
    q = rng.standard_normal((B, N, Hq, d))
    k = rng.standard_normal((B, N, Hkv, d))
    v = rng.standard_normal((B, N, Hkv, d))
    wc, _ = oracle.cutoffs(d, 30.0, oracle.HALF_SPLIT)
    assert len(set(np.asarray(wc).tolist())) > 3  # several distinct windows inside N
    C = d // 2
    perm = np.empty(d, dtype=np.int64)
    perm[0::2], perm[1::2] = np.arange(C), np.arange(C) + C
    o1, l1 = oracle.attention(q, k, v, wc, oracle.MODE_CHANNEL, oracle.HALF_SPLIT)
    o2, l2 = oracle.attention(q[..., perm], k[..., perm], v, wc, oracle.MODE_CHANNEL, oracle.INTERLEAVED)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(l2, l1, rtol=1e-12, atol=1e-12)
    # and the paired order's groups are the interleaved groups: each holds 8
    # whole channels, so its cutoff is the largest of those 8 channel cutoffs
    wc_i, wg_i = oracle.cutoffs(d, 30.0, oracle.INTERLEAVED)
    assert np.array_equal(np.asarray(wc_i), np.asarray(wc))
    assert wg_i[0] == max(wc[:8]) and wg_i[1] == max(wc[8:])


# --------------------------------------------------------------------------
# Backward: gradients of the prefill definition
# --------------------------------------------------------------------------

def _bwd_case(seed, N=17, Hq=2, Hkv=1, d=32):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, N, Hq, d))
    k = rng.standard_normal((1, N, Hkv, d))
    v = rng.standard_normal((1, N, Hkv, d))
    dout = rng.standard_normal((1, N, Hq, d))
    return q, k, v, dout


BWD_CASES = [
    # mode, layout, cutoffs (small, so masks bite at distances < N)
    (oracle.MODE_GROUPED, oracle.INTERLEAVED, [3, 9]),
    (oracle.MODE_GROUPED, oracle.HALF_SPLIT, [0, 5]),
    (oracle.MODE_CHANNEL, oracle.INTERLEAVED, [0, 1, 2, 3, 5, 7, 9, 12, 2, 4, 6, 8, 10, 11, 13, 20]),
    (oracle.MODE_CHANNEL, oracle.HALF_SPLIT, [1, 3, 0, 6, 2, 8, 4, 11, 5, 7, 3, 9, 14, 2, 6, 10]),
]


@pytest.mark.parametrize("mode,layout,cut", BWD_CASES)
def test_backward_central_differences(mode, layout, cut):
    """Each gradient entry equals the central difference of the loss
    sum(dout * O) computed with the oracle's forward pass (itself pinned to
    SDPA, closed forms and invariants above): fp64, step 1e-6, on a random
    subset of entries of q, k and v (GQA: two query heads per KV head)."""
    cut = np.asarray(cut, dtype=np.int32)
    q, k, v, dout = _bwd_case(7)
    dq, dk, dv = oracle.attention_backward(q, k, v, dout, cut, mode, layout)

    def loss(q_, k_, v_):
        o, _ = oracle.attention(q_, k_, v_, cut, mode, layout)
        return float((o * dout).sum())

    rng = np.random.default_rng(1)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in zip(*[rng.integers(0, s, 25) for s in x.shape]):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - g[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, g[idx])


def _torch_wave_attention(q, k, v, cut, mode, layout):
    """Independent torch statement of the forward rule: per-unit masked
    logits summed, causal -inf, softmax, times V. q [N,Hq,d], k/v [N,Hkv,d]."""
    N, Hq, d = q.shape
    Hkv = k.shape[1]
    rep = Hq // Hkv
    kk = k.repeat_interleave(rep, dim=1)
    vv = v.repeat_interleave(rep, dim=1)
    dist = torch.arange(N)[:, None] - torch.arange(N)[None, :]
    if mode == oracle.MODE_GROUPED:
        units = [list(range(16 * g, 16 * g + 16)) for g in range(d // 16)]
    elif layout == oracle.INTERLEAVED:
        units = [[2 * c, 2 * c + 1] for c in range(d // 2)]
    else:
        units = [[c, c + d // 2] for c in range(d // 2)]
    L = torch.zeros(Hq, N, N, dtype=q.dtype)
    for u, dims in enumerate(units):
        part = torch.einsum("ihe,jhe->hij", q[:, :, dims], kk[:, :, dims])
        L = L + part * (dist <= int(cut[u])).to(q.dtype)
    L = L / math.sqrt(d)
    L = L.masked_fill(dist < 0, float("-inf"))
    return torch.einsum("hij,jhe->ihe", torch.softmax(L, dim=-1), vv)


@pytest.mark.parametrize("mode,layout,cut", BWD_CASES)
def test_backward_matches_torch_autograd(mode, layout, cut):
    """torch autograd through an independently written torch statement of the
    same rule gives the oracle's gradients (fp64), including the sum over the
    query heads that share a KV head."""
    q, k, v, dout = _bwd_case(11, N=23, Hq=4, Hkv=2)
    cut = np.asarray(cut, dtype=np.int32)
    dq, dk, dv = oracle.attention_backward(q, k, v, dout, cut, mode, layout)
    tq, tk, tv = (torch.tensor(x[0], requires_grad=True) for x in (q, k, v))
    o = _torch_wave_attention(tq, tk, tv, cut, mode, layout)
    (o * torch.tensor(dout[0])).sum().backward()
    for name, mine, ref in (("dq", dq, tq.grad), ("dk", dk, tk.grad), ("dv", dv, tv.grad)):
        np.testing.assert_allclose(mine[0], ref.numpy(), rtol=0, atol=1e-10, err_msg=name)


def test_backward_dense_is_sdpa_autograd():
    """[RN §2.1]: alpha -> infinity (every cutoff >= N) is plain causal
    attention, whose gradients torch's scaled_dot_product_attention gives."""
    q, k, v, dout = _bwd_case(3, N=30, Hq=4, Hkv=2, d=64)
    for mode, n in ((oracle.MODE_GROUPED, 4), (oracle.MODE_CHANNEL, 32)):
        dq, dk, dv = oracle.attention_backward(q, k, v, dout, np.full(n, 2 ** 31 - 1, dtype=np.int32), mode,
                                               oracle.INTERLEAVED)
        tq, tk, tv = (torch.tensor(x[0].transpose(1, 0, 2), requires_grad=True) for x in (q, k, v))
        o = torch.nn.functional.scaled_dot_product_attention(tq, tk.repeat_interleave(2, 0),
                                                             tv.repeat_interleave(2, 0), is_causal=True)
        (o * torch.tensor(dout[0].transpose(1, 0, 2))).sum().backward()
        for name, mine, ref in (("dq", dq, tq.grad), ("dk", dk, tk.grad), ("dv", dv, tv.grad)):
            np.testing.assert_allclose(mine[0], ref.numpy().transpose(1, 0, 2), rtol=0, atol=1e-10,
                                       err_msg=f"{name} mode={mode}")
