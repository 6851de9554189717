"""GPU parity of wp_prefill_backward (grouped mode) against the fp64
oracle's gradients, on the same bf16 inputs: ragged lengths, GQA, boundary
cutoffs inside tiles, per-head tables, dense and all-zero tables."""
import numpy as np
import pytest
import torch

import oracle
import rope_period_truncated_b200 as wp
import wp_synthetic as syn
from parity import assert_grad_close, widen

pytestmark = pytest.mark.gpu


def _run(q, k, v, dout, cut, layout, mode=wp.MODE_GROUPED):
    qg, kg, vg, dg = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    o, lse = wp.wp_prefill(qg, kg, vg, cut, mode, layout)
    dq, dk, dv = wp.wp_prefill_backward(qg, kg, vg, o, lse, dg, cut)
    torch.cuda.synchronize()
    assert wp.wp_device_status() == 0
    return dq, dk, dv


def _check(q, k, v, dout, cut, layout, tag):
    dq, dk, dv = _run(q, k, v, dout, cut, layout)
    d = q.shape[-1]
    ocut = cut if cut is not None else np.full(d // 16, 2 ** 31 - 1, dtype=np.int32)
    if np.asarray(ocut).ndim == 2:  # per-head rows: the oracle one head at a time
        Hq, Hkv = q.shape[2], k.shape[2]
        rdq = np.zeros(q.shape)
        rdk = np.zeros(k.shape)
        rdv = np.zeros(v.shape)
        for h in range(Hq):
            hk = h // (Hq // Hkv)
            a, b_, c = oracle.attention_backward(widen(q[:, :, h:h + 1]), widen(k[:, :, hk:hk + 1]),
                                                 widen(v[:, :, hk:hk + 1]), widen(dout[:, :, h:h + 1]), ocut[h],
                                                 oracle.MODE_GROUPED, layout)
            rdq[:, :, h:h + 1] = a
            rdk[:, :, hk:hk + 1] += b_
            rdv[:, :, hk:hk + 1] += c
    else:
        rdq, rdk, rdv = oracle.attention_backward(widen(q), widen(k), widen(v), widen(dout), ocut,
                                                  oracle.MODE_GROUPED, layout)
    assert_grad_close(dq, rdq, f"{tag} dq")
    assert_grad_close(dk, rdk, f"{tag} dk")
    assert_grad_close(dv, rdv, f"{tag} dv")


def _draw(seed, B, N, Hq, Hkv, d):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, N, Hq, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, N, Hkv, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, N, Hkv, d, generator=g).to(torch.bfloat16)
    dout = torch.randn(B, N, Hq, d, generator=g).to(torch.bfloat16)
    return q, k, v, dout


def test_tiny_workload_backward():
    """Tiny workload (B1 H2/2 N256 d64 theta 1e4 interleaved), rotated inputs."""
    w = syn.workload("tiny")
    q, k, v = syn.prefill_inputs(w)
    q = wp.wp_rope_apply(q.cuda(), w.theta, w.layout).cpu()
    k = wp.wp_rope_apply(k.cuda(), w.theta, w.layout).cpu()
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16)
    _, wg = oracle.cutoffs(w.d, w.theta, w.layout)
    _check(q, k, v, dout, wg, w.layout, "tiny")


SHAPES = [
    # N, d, Hq, Hkv, layout, table
    (1, 128, 2, 1, wp.ROPE_HALF_SPLIT, "wave"),
    (127, 64, 2, 2, wp.ROPE_INTERLEAVED, "wave"),
    (129, 128, 4, 2, wp.ROPE_HALF_SPLIT, "mixed"),
    (300, 128, 6, 2, wp.ROPE_INTERLEAVED, "wave"),   # 3 query heads per KV head
    (513, 64, 4, 1, wp.ROPE_HALF_SPLIT, "mixed"),
    (200, 128, 2, 2, wp.ROPE_HALF_SPLIT, "zero"),
    (200, 128, 4, 2, wp.ROPE_HALF_SPLIT, "dense"),
    (333, 128, 4, 2, wp.ROPE_HALF_SPLIT, "per_head"),
]


def _table(kind, d, Hq, theta, layout):
    G = d // 16
    if kind == "wave":
        return oracle.cutoffs(d, theta, layout)[1]
    if kind == "mixed":
        return np.resize(np.array([0, 3, 130, 40, 50, 200, 65, 1000], dtype=np.int32), G)
    if kind == "zero":
        return np.zeros(G, dtype=np.int32)
    if kind == "dense":
        return None
    if kind == "per_head":
        rng = np.random.default_rng(Hq)
        return rng.integers(0, 300, size=(Hq, G)).astype(np.int32)
    raise ValueError(kind)


@pytest.mark.parametrize("N,d,Hq,Hkv,layout,kind", SHAPES)
def test_backward_small_shapes(N, d, Hq, Hkv, layout, kind):
    q, k, v, dout = _draw(500 + N + d, 2, N, Hq, Hkv, d)
    cut = _table(kind, d, Hq, 1e4, layout)
    _check(q, k, v, dout, cut, layout, f"N={N} d={d} Hq={Hq} Hkv={Hkv} {kind}")


def test_backward_4k_qwen_shaped_heads():
    """4K context with the Qwen3-8B head shape (d128, theta 1e6, half-split,
    GQA 4:1) on 4 query heads: every gradient entry against the oracle."""
    w = syn.workload("qwen3_8b_4k")
    q, k, v, dout = _draw(41, 1, 4096, 4, 1, 128)
    _, wg = oracle.cutoffs(w.d, w.theta, w.layout)
    _check(q, k, v, dout, wg, w.layout, "4k")
