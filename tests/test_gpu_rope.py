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
