"""The bench's work accounting (useful FLOPs, required decode bytes, the ncu
traffic lookup) checked against brute-force enumeration on small cases and
against the figures the scope table states for the 32K workload. Host only."""
import os

import numpy as np
import pytest

import bench


def _brute_pair_exact(N, d, wg):
    total = 0
    for i in range(N):
        for j in range(i + 1):
            total += 2 * 16 * sum(1 for w in wg if i - j <= w) + 2 * d
    return total


def _brute_tile_level(N, d, wg, BM=128, BN=128):
    total = 0
    nqb = (N + BM - 1) // BM
    for qb in range(nqb):
        qs, qe = qb * BM, min(qb * BM + BM, N) - 1
        for kb in range(qb + 1):
            ks, ke = kb * BN, min(kb * BN + BN, N) - 1
            if ks > qe:
                continue
            dmax, dmin = qe - ks, (qs - ke if qs > ke else 0)
            live = sum(1 for w in wg if dmin <= w)  # not skipped: full or boundary
            total += live * 2 * BM * BN * 16 + 2 * BM * BN * d
    return total


@pytest.mark.parametrize("N", [1, 127, 300, 513])
def test_prefill_flops_match_enumeration(N):
    d, wg = 64, [0, 3, 130, 1000]
    tile, pair, dense = bench.prefill_flops(N, d, 2, 3, wg)
    assert pair == _brute_pair_exact(N, d, wg) * 2 * 3
    assert tile == _brute_tile_level(N, d, wg) * 2 * 3
    assert dense == _brute_tile_level(N, d, [10 ** 9] * (d // 16)) * 2 * 3  # every group kept


def test_prefill_flops_32k_figures():
    """Scope table: 6.922 TFLOP pair-exact useful work for the 32K prefill, and
    8.796 TFLOP dense causal (same count with every group kept)."""
    wg = [160, 5063, 160114, 5063255] * 2
    _, pair, _ = bench.prefill_flops(32768, 128, 32, 1, wg)
    _, pair_dense, _ = bench.prefill_flops(32768, 128, 32, 1, [2 ** 31 - 1] * 8)
    assert abs(pair / 1e12 - 6.922) < 5e-4
    assert abs(pair_dense / 1e12 - 8.796) < 5e-4


@pytest.mark.parametrize("N", [1, 130, 400])
def test_backward_flops_match_enumeration(N):
    """Per causal pair: S, dQ and dK over the in-window groups (2*16 each per
    group) and dP, dV in full (2*d each)."""
    d, wg = 64, [0, 3, 130, 1000]
    useful, dense = bench.backward_flops(N, d, 2, 3, wg)
    tot = tot_dense = 0
    for i in range(N):
        for j in range(i + 1):
            tot += 3 * 2 * 16 * sum(1 for w in wg if i - j <= w) + 2 * 2 * d
            tot_dense += 3 * 2 * d + 2 * 2 * d
    assert useful == tot * 2 * 3
    assert dense == tot_dense * 2 * 3


@pytest.mark.parametrize("N", [1, 130, 400])
def test_exact_flops_match_enumeration(N):
    """Per causal pair: 2*2 per channel with i-j <= W_c (its two dims) and
    2*d for PV; every channel kept gives the dense causal count."""
    d = 64
    wc = [0, 3, 7, 130, 131, 1000] + [2 ** 31 - 1] * (d // 2 - 6)
    tot = 0
    for i in range(N):
        for j in range(i + 1):
            tot += 2 * 2 * sum(1 for w in wc if i - j <= w) + 2 * d
    assert bench.exact_flops(N, d, 2, 3, wc) == tot * 2 * 3
    dense = sum(4 * d for i in range(N) for j in range(i + 1)) * 2 * 3
    assert bench.exact_flops(N, d, 2, 3, [2 ** 31 - 1] * (d // 2)) == dense


def test_decode_required_bytes_match_enumeration():
    rng = np.random.default_rng(3)
    lens = rng.integers(1, 400, size=5)
    wg = [2, 17, 100, 10 ** 6]
    B, Hq, Hkv, d = 5, 8, 2, 64
    req, dense = bench.decode_required_bytes(lens, wg, B, Hq, Hkv, d)
    kv = 0
    for L in lens:
        q = L - 1
        for j in range(L):
            kv += 32 * sum(1 for w in wg if q - j <= w) + 2 * d  # K of in-window groups + V row
    io = B * Hq * d * 2 * 2 + B * Hq * 4
    assert req == kv * Hkv + io
    assert dense == sum(4 * d * L for L in lens) * Hkv + io


def test_profiled_traffic_follows_the_source(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.source_digest("kernel.cu")
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "k.txt").write_text(
        f"# comment: with a colon\nsource_sha256_16: {h}\ndram_bytes_per_launch: 12345\n")
    assert bench.profiled_traffic("k.txt", "kernel.cu") == 12345
    src.write_text("kernel v2\n")  # the kernel changed since the capture
    assert bench.profiled_traffic("k.txt", "kernel.cu") is None
    assert bench.profiled_traffic("missing.txt", "kernel.cu") is None


def test_source_digest_covers_included_headers(tmp_path, monkeypatch):
    """A change to a header the kernel includes (beside it or in include/)
    changes the digest; an unrelated file does not."""
    (tmp_path / "csrc").mkdir()
    (tmp_path / "include").mkdir()
    (tmp_path / "csrc" / "k.cu").write_text('#include "a.cuh"\n#include <cstdint>\nkernel\n')
    (tmp_path / "csrc" / "a.cuh").write_text('#include "api.h"\n#include "a.cuh"\nhelpers v1\n')
    (tmp_path / "include" / "api.h").write_text("api v1\n")
    (tmp_path / "csrc" / "other.cuh").write_text("unrelated v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    d0 = bench.source_digest("csrc/k.cu")
    assert len(d0) == 16
    (tmp_path / "csrc" / "other.cuh").write_text("unrelated v2\n")
    assert bench.source_digest("csrc/k.cu") == d0
    (tmp_path / "csrc" / "a.cuh").write_text('#include "api.h"\n#include "a.cuh"\nhelpers v2\n')
    d1 = bench.source_digest("csrc/k.cu")
    assert d1 != d0
    (tmp_path / "include" / "api.h").write_text("api v2\n")
    d2 = bench.source_digest("csrc/k.cu")
    assert d2 not in (d0, d1)
    # comments and whitespace are not compiled: editing them keeps the digest
    (tmp_path / "include" / "api.h").write_text("// a note\napi   v2 /* more\n notes */\n")
    assert bench.source_digest("csrc/k.cu") == d2
