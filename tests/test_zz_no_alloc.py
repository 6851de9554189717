"""wp_decode_static: decode for callers that cannot allocate device memory
(e.g. an engine whose device memory is planned up front and served by its own
pool, or a decode loop that must not reach cudaMalloc/cudaFree). Its split
partials live in the library's fixed 16 MiB device scratch instead of a
caller workspace. Checked through the C ABI against the fp64 oracle and
against wp_decode on the same inputs, on three calls in a row (each reuses
the scratch the one before left behind; the second has the first one's shape
with fewer active splits), and for the size limit.

This file is collected last so that a run stopping at the first failure has
already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import rope_period_truncated_b200 as wp
from parity import LSE_REL, O_MAX_ABS, O_MEAN_ABS, assert_attention_close, widen

pytestmark = pytest.mark.gpu


def _inputs(seed, B, Hq, Hkv, d, Lmax, lens):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16).cuda()
    kc = torch.randn(B, Hkv, Lmax, d, generator=g).to(torch.bfloat16).cuda()
    vc = torch.randn(B, Hkv, Lmax, d, generator=g).to(torch.bfloat16).cuda()
    return q, kc, vc, torch.tensor(lens, dtype=torch.int32, device="cuda")


def _call_static(lib, q, kc, vc, lens, cut, o, lse):
    B, Hq, d = q.shape
    _, Hkv, Lmax, _ = kc.shape
    cut_a = np.ascontiguousarray(cut, dtype=np.int32)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return lib.wp_decode_static(p(q), p(kc), p(vc), p(lens), Lmax, B, Hq, Hkv, d,
                                cut_a.ctypes.data_as(ctypes.c_void_p), ctypes.c_float(0.0), p(o), p(lse),
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _close(o_a, l_a, o_b, l_b):
    err = (o_a.float() - o_b.float()).abs()
    assert err.max().item() <= O_MAX_ABS and err.mean().item() <= O_MEAN_ABS
    lerr = (l_a - l_b).abs()
    assert (lerr <= LSE_REL * torch.clamp(l_b.abs(), min=1.0)).all()


def test_static_scratch_decode_matches_oracle_and_workspace_decode():
    """Three calls in a row on the one scratch array: a long batch, then the
    same shape with shorter sequences (fewer splits hold keys, so stale
    partials of the first call sit beyond the active ones), then another
    shape. Each result is checked against the fp64 oracle and against
    wp_decode with a caller workspace."""
    lib = wp.load_library()
    _, wg = oracle.cutoffs(128, 1e6, oracle.HALF_SPLIT)
    cases = [
        (31, 4, 8, 2, 128, 3000, [1, 2999, 1500, 3000]),
        (33, 4, 8, 2, 128, 3000, [700, 1, 100, 1025]),
        (32, 3, 16, 2, 128, 5000, [4999, 7, 2048]),
    ]
    for seed, B, Hq, Hkv, d, Lmax, lens in cases:
        q, kc, vc, ln = _inputs(seed, B, Hq, Hkv, d, Lmax, lens)
        o_ref, l_ref = wp.wp_decode(q, kc, vc, ln, wg)
        o = torch.empty_like(q)
        lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
        assert _call_static(lib, q, kc, vc, ln, wg, o, lse) == wp.WP_OK
        torch.cuda.synchronize()
        assert wp.wp_device_status() == wp.WP_OK
        _close(o, lse, o_ref, l_ref)
        ro, rl = oracle.decode(widen(q), widen(kc), widen(vc), np.asarray(lens, dtype=np.int32), wg)
        assert_attention_close(o, lse, ro, rl, f"static decode lens={lens}")


def test_static_scratch_rejects_oversized_batch():
    """A batch whose partials exceed the fixed scratch is refused up front."""
    lib = wp.load_library()
    B, Hq, Hkv, d, Lmax = 64, 64, 8, 128, 131072
    assert wp.wp_decode_workspace_bytes(B, Hq, d, Lmax) > wp.DECODE_STATIC_SCRATCH_BYTES
    t = torch.empty(16, dtype=torch.bfloat16, device="cuda")  # never read: nothing is launched
    p = ctypes.c_void_p(t.data_ptr())
    rc = lib.wp_decode_static(p, p, p, p, Lmax, B, Hq, Hkv, d, None, ctypes.c_float(0.0), p, p,
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == wp.WP_ERR_UNSUPPORTED
