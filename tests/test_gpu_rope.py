"""GPU parity of wp_rope_apply against the oracle's fp64 rotation rounded to
bf16 (at most 1 ulp apart; nearly all elements bit-identical)."""
import numpy as np
import pytest
import torch

import oracle
import rope_period_truncated_b200 as wp
import wp_synthetic as syn
from parity import bf16_bits, ulp_distance, widen

pytestmark = pytest.mark.gpu


def _pair_magnitude(x, layout):
    """|x_a| + |x_b| of the channel pair every element belongs to."""
    C = x.shape[-1] // 2
    m = np.empty_like(x)
    if layout == wp.ROPE_INTERLEAVED:
        pm = np.abs(x[..., 0::2]) + np.abs(x[..., 1::2])
        m[..., 0::2], m[..., 1::2] = pm, pm
    else:
        pm = np.abs(x[..., :C]) + np.abs(x[..., C:])
        m[..., :C], m[..., C:] = pm, pm
    return m


def _check(y_gpu, x_cpu, theta, layout, pos=None, pos0=0, scale_all=1.0, freq_scale=None):
    """The kernel rotates in fp32, so its result is the bf16 rounding of a
    value within a few fp32 ulps of the pair's magnitude of the exact
    rotation. Away from cancellation that is at most 1 bf16 ulp; where
    x_a cos - x_b sin nearly cancels, the absolute fp32 bound applies."""
    x = widen(x_cpu)
    ref = oracle.rope(x, theta, layout, pos=pos, pos0=pos0, scale_all=scale_all, freq_scale=freq_scale)
    ref_bits = oracle.round_bf16_bits(ref)
    ulps = ulp_distance(bf16_bits(y_gpu), ref_bits)
    mag = _pair_magnitude(x, layout)
    y = widen(y_gpu)
    ulp_ref = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    err = np.abs(y - ref)
    assert np.all(err <= ulp_ref + 2.0 ** -20 * mag), f"max excess {np.max(err - ulp_ref - 2.0 ** -20 * mag):.3e}"
    clean = np.abs(ref) >= 2.0 ** -8 * mag  # no heavy cancellation
    assert ulps[clean].max() <= 1, f"max ulp distance {ulps[clean].max()} away from cancellation"
    assert (ulps > 0).mean() < 0.02, f"{(ulps > 0).mean():.3%} elements differ"


@pytest.mark.parametrize("layout", [wp.ROPE_INTERLEAVED, wp.ROPE_HALF_SPLIT])
@pytest.mark.parametrize("d", [64, 128])
def test_rope_small(layout, d):
    g = torch.Generator().manual_seed(11)
    x = torch.randn(2, 301, 3, d, generator=g).to(torch.bfloat16)
    y = wp.wp_rope_apply(x.cuda(), 1e4 if d == 64 else 1e6, layout)
    torch.cuda.synchronize()
    _check(y, x, 1e4 if d == 64 else 1e6, layout)


@pytest.mark.parametrize("layout", [wp.ROPE_INTERLEAVED, wp.ROPE_HALF_SPLIT])
def test_rope_positions_offset_scale_inplace(layout):
    g = torch.Generator().manual_seed(12)
    x = torch.randn(2, 257, 4, 128, generator=g).to(torch.bfloat16)
    pos = torch.randint(0, 1 << 21, (2, 257), generator=g, dtype=torch.int32)
    xg = x.cuda()
    y = wp.wp_rope_apply(xg, 1e6, layout, pos=pos.cuda(), scale_all=0.25, out=xg)  # in place
    torch.cuda.synchronize()
    assert y.data_ptr() == xg.data_ptr()
    _check(y, x, 1e6, layout, pos=pos.numpy(), scale_all=0.25)
    y2 = wp.wp_rope_apply(x.cuda(), 1e6, layout, pos0=98765)
    torch.cuda.synchronize()
    _check(y2, x, 1e6, layout, pos0=98765)
    fs = np.linspace(0.3, 1.0, 64)
    y3 = wp.wp_rope_apply(x.cuda(), 1e6, layout, freq_scale=fs)
    torch.cuda.synchronize()
    _check(y3, x, 1e6, layout, freq_scale=fs)


@pytest.mark.parametrize("name", ["long_32k", "scaled_128k"])
def test_rope_full_size_sampled_tokens(name):
    """Full-size Q rotation (the bench's launch), checked on 512 sampled tokens."""
    w = syn.workload(name)
    q, _, _ = syn.prefill_inputs(w)
    y = wp.wp_rope_apply(q.cuda(), w.theta, w.layout, scale_all=w.scale_all)
    torch.cuda.synchronize()
    g = torch.Generator().manual_seed(13)
    tok = torch.randint(0, w.N, (512,), generator=g)
    tok[-1] = w.N - 1
    xs = q[0, tok].unsqueeze(0)          # [1, 512, H, d]
    ys = y[0, tok.cuda()].unsqueeze(0)
    _check(ys, xs, w.theta, w.layout, pos=tok.numpy().reshape(1, -1), scale_all=w.scale_all)


def _paired_perm(d):
    """Output dim 2c takes half-split dim c, dim 2c+1 takes dim c + d/2."""
    C = d // 2
    perm = np.empty(d, dtype=np.int64)
    perm[0::2] = np.arange(C)
    perm[1::2] = np.arange(C) + C
    return perm


@pytest.mark.parametrize("d", [64, 128])
def test_rope_half_split_paired_is_a_permutation(d):
    """WP_ROPE_HALF_SPLIT_PAIRED is the half-split rotation with channel c's
    pair moved to dims (2c, 2c+1): bit-identical to permuting the half-split
    result."""
    g = torch.Generator().manual_seed(50 + d)
    x = torch.randn(2, 300, 3, d, generator=g).to(torch.bfloat16).cuda()
    pos = torch.randint(0, 40000, (2, 300), generator=g).to(torch.int32).cuda()
    hs = wp.wp_rope_apply(x, 1e6, wp.ROPE_HALF_SPLIT, pos=pos)
    pr = wp.wp_rope_apply(x, 1e6, wp.ROPE_HALF_SPLIT_PAIRED, pos=pos)
    torch.cuda.synchronize()
    perm = torch.from_numpy(_paired_perm(d)).cuda()
    assert torch.equal(pr, hs[..., perm])


def test_prefill_paired_grouping_matches_oracle():
    """Paper-equivalent grouping of a half-split model: Q and K rotated into
    the interleaved order, then the interleaved group cutoffs (8 whole
    channels per group, [RN §2.3, Table 12]). The oracle rotates half-split
    in fp64, permutes the same way and applies the grouped rule with the
    interleaved cutoffs."""
    g = torch.Generator().manual_seed(77)
    B, N, Hq, Hkv, d, theta = 1, 700, 4, 2, 128, 1e6
    q = torch.randn(B, N, Hq, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, N, Hkv, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, N, Hkv, d, generator=g).to(torch.bfloat16)
    _, wg = oracle.cutoffs(d, theta, oracle.INTERLEAVED)
    wg = np.asarray(wg) // 40  # shrink the windows so that N = 700 spans several cutoffs
    wg = np.maximum(wg, 0).astype(np.int32)
    qp = wp.wp_rope_apply(q.cuda(), theta, wp.ROPE_HALF_SPLIT_PAIRED)
    kp = wp.wp_rope_apply(k.cuda(), theta, wp.ROPE_HALF_SPLIT_PAIRED)
    o, lse = wp.wp_prefill(qp, kp, v.cuda(), wg, wp.MODE_GROUPED, wp.ROPE_INTERLEAVED)
    torch.cuda.synchronize()
    assert wp.wp_device_status() == 0
    perm = _paired_perm(d)
    qo = oracle.bf16_bits_to_f64(oracle.round_bf16_bits(oracle.rope(widen(q), theta, oracle.HALF_SPLIT)))[..., perm]
    ko = oracle.bf16_bits_to_f64(oracle.round_bf16_bits(oracle.rope(widen(k), theta, oracle.HALF_SPLIT)))[..., perm]
    ro, rl = oracle.attention(qo, ko, widen(v), wg, oracle.MODE_GROUPED, oracle.INTERLEAVED)
    from parity import assert_attention_close
    assert_attention_close(o, lse, ro, rl, "paired grouping")
