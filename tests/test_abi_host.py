"""C-ABI checks that need no GPU: the library loads, exports every symbol
the header declares, the host-only calls (cutoff tables, tile schedule) are
bit-exact against the fp64 oracle, and argument checks reject bad calls
before anything is launched."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import rope_period_truncated_b200 as wp
from rope_period_truncated_b200 import build as wpbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    wpbuild.build()
    return wp.load_library()


def test_exports_every_declared_symbol(lib):
    header = open(os.path.join(ROOT, "include", "waveprune.h")).read()
    declared = set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(wp_\w+)\s*\(", header, re.M))
    assert {"wp_cutoffs", "wp_rope_apply", "wp_schedule", "wp_prefill", "wp_decode"} <= declared
    for name in declared:
        assert hasattr(lib, name), name


CUTOFF_CASES = [
    (64, 1e4, wp.ROPE_INTERLEAVED, 1.0, 2.0),
    (64, 1e4, wp.ROPE_HALF_SPLIT, 1.0, 2.0),
    (128, 1e6, wp.ROPE_HALF_SPLIT, 1.0, 2.0),
    (128, 1e6, wp.ROPE_INTERLEAVED, 1.0, 2.0),
    (128, 1e6, wp.ROPE_HALF_SPLIT, 0.25, 2.0),
    (128, 5e5, wp.ROPE_HALF_SPLIT, 1.0, 1.5),
    (64, 1e4, wp.ROPE_INTERLEAVED, 1.0, 1e300),
]


@pytest.mark.parametrize("d,theta,layout,scale_all,alpha", CUTOFF_CASES)
def test_cutoffs_bit_exact(lib, d, theta, layout, scale_all, alpha):
    a_c, a_g = wp.wp_cutoffs(d, theta, layout, alpha=alpha, scale_all=scale_all)
    b_c, b_g = oracle.cutoffs(d, theta, layout, alpha=alpha, scale_all=scale_all)
    assert np.array_equal(a_c, b_c) and np.array_equal(a_g, b_g)


def test_cutoffs_per_channel_scale(lib):
    rng = np.random.default_rng(0)
    fs = rng.uniform(0.2, 1.0, 64)
    a = wp.wp_cutoffs(128, 1e6, wp.ROPE_HALF_SPLIT, freq_scale=fs)
    b = oracle.cutoffs(128, 1e6, oracle.HALF_SPLIT, freq_scale=fs)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_cutoffs_reject_bad_arguments(lib):
    out = np.zeros(64, dtype=np.int32)
    p = out.ctypes.data_as(ctypes.c_void_p)
    assert lib.wp_cutoffs(100, 1e4, None, 1.0, 2.0, 0, p, p) == wp.WP_ERR_ARG    # d_h not a multiple of 16
    assert lib.wp_cutoffs(64, 1.0, None, 1.0, 2.0, 0, p, p) == wp.WP_ERR_ARG     # theta <= 1
    assert lib.wp_cutoffs(64, 1e4, None, 0.0, 2.0, 0, p, p) == wp.WP_ERR_ARG     # scale <= 0
    assert lib.wp_cutoffs(64, 1e4, None, float("nan"), 2.0, 0, p, p) == wp.WP_ERR_ARG
    assert lib.wp_cutoffs(64, 1e4, None, 1.0, 0.0, 0, p, p) == wp.WP_ERR_ARG     # alpha <= 0
    assert lib.wp_cutoffs(64, 1e4, None, 1.0, 2.0, 7, p, p) == wp.WP_ERR_ARG     # layout


SCHEDULE_CASES = [(256, 128, 128), (300, 128, 128), (4096, 128, 128), (1000, 64, 128), (777, 128, 64), (1, 128, 128),
                  (129, 128, 128)]


@pytest.mark.parametrize("N,BM,BN", SCHEDULE_CASES)
def test_schedule_bit_exact_vs_brute_force(lib, N, BM, BN):
    cuts = [0, 5, 28, 127, 128, 160, 255, 256, 900, 5063, 2 ** 31 - 1]
    a_cls, a_cnt = wp.wp_schedule(N, BM, BN, cuts)
    b_cls, b_cnt = oracle.tile_classes(N, BM, BN, cuts)
    assert np.array_equal(a_cls, b_cls)
    assert np.array_equal(a_cnt, b_cnt)


@pytest.mark.parametrize("name,N", [("long_32k", 32768), ("qwen3_8b_4k", 4096)])
def test_schedule_workload_counts(lib, name, N):
    """Bit-exact per-group counts for the benchmark workloads' own cutoffs."""
    _, wg = oracle.cutoffs(128, 1e6, oracle.HALF_SPLIT)
    _, a_cnt = wp.wp_schedule(N, 128, 128, wg, want_map=False)
    _, b_cnt = oracle.tile_classes(N, 128, 128, wg, want_map=False)
    assert np.array_equal(a_cnt, b_cnt)


def test_schedule_rejects_bad_arguments(lib):
    cut = np.zeros(4, dtype=np.int32)
    cnt = np.zeros(12, dtype=np.int64)
    cp, np_ = cut.ctypes.data_as(ctypes.c_void_p), cnt.ctypes.data_as(ctypes.c_void_p)
    assert lib.wp_schedule(0, 128, 128, cp, 4, None, np_) == wp.WP_ERR_ARG
    assert lib.wp_schedule(10, 0, 128, cp, 4, None, np_) == wp.WP_ERR_ARG
    assert lib.wp_schedule(10, 128, 128, None, 4, None, np_) == wp.WP_ERR_ARG
    neg = np.array([-1], dtype=np.int32)
    assert lib.wp_schedule(10, 128, 128, neg.ctypes.data_as(ctypes.c_void_p), 1, None, np_) == wp.WP_ERR_ARG


# Device calls: every case below breaks a rule that is checked on the host
# before any CUDA call, so nothing is launched (safe with or without a GPU).
FAKE = 1 << 20  # a 16-byte aligned fake address, never dereferenced


def test_prefill_rejects_bad_arguments(lib):
    cut = (ctypes.c_int32 * 8)(*([100] * 8))
    f = lib.wp_prefill
    ok = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, B=1, N=64, Hq=4, Hkv=2, d=128, mode=0, layout=1)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["N"], a["Hq"], a["Hkv"], a["d"], a["mode"],
                 cut, a["layout"], ctypes.c_float(0.0), None)

    assert call(q=None) == wp.WP_ERR_ARG
    assert call(o=FAKE + 8) == wp.WP_ERR_ARG          # misaligned
    assert call(Hq=3) == wp.WP_ERR_ARG                # Hq % Hkv
    assert call(N=0) == wp.WP_ERR_ARG
    assert call(d=96) == wp.WP_ERR_UNSUPPORTED
    assert call(d=100) == wp.WP_ERR_ARG
    assert call(mode=5) == wp.WP_ERR_ARG
    assert call(N=(1 << 20) + 1) == wp.WP_ERR_UNSUPPORTED  # key-block table beyond shared memory
    assert call(layout=3) == wp.WP_ERR_ARG
    negcut = (ctypes.c_int32 * 8)(*([-1] * 8))
    assert f(FAKE, FAKE, FAKE, FAKE, None, 1, 64, 4, 2, 128, 0, negcut, 1, ctypes.c_float(0.0), None) == wp.WP_ERR_ARG
    assert f(FAKE, FAKE, FAKE, FAKE, None, 1, 64, 4, 2, 128, 0, cut, 1, ctypes.c_float(float("inf")),
             None) == wp.WP_ERR_ARG


def test_decode_rejects_bad_arguments(lib):
    f = lib.wp_decode
    ws = lib.wp_decode_workspace_bytes(2, 8, 128, 4096)
    assert ws > 0
    args = [FAKE, FAKE, FAKE, FAKE, 4096, 2, 8, 2, 128, None, ctypes.c_float(0.0), FAKE, None, FAKE, ws, None]

    def call(i, val):
        a = list(args)
        a[i] = val
        return f(*a)

    assert call(0, None) == wp.WP_ERR_ARG               # q NULL
    assert call(13, FAKE + 16) == wp.WP_ERR_ARG         # workspace not 256-aligned
    assert call(14, ws - 1) == wp.WP_ERR_ARG            # workspace too small
    assert call(6, 6) == wp.WP_ERR_UNSUPPORTED          # 3 query heads per KV head
    assert call(8, 72) == wp.WP_ERR_ARG                 # d_h not a multiple of 16
    assert call(8, 80) == wp.WP_ERR_UNSUPPORTED         # d_h not 64 or 128
    assert call(4, 0) == wp.WP_ERR_ARG                  # Lmax


def test_decode_kl_and_kcache_conversion_reject_bad_arguments(lib):
    f = lib.wp_decode_kl
    ws = lib.wp_decode_workspace_bytes(2, 8, 128, 4096)
    args = [FAKE, FAKE, wp.KCACHE_GROUP_MAJOR, FAKE, FAKE, 4096, 2, 8, 2, 128, None, ctypes.c_float(0.0), FAKE,
            None, FAKE, ws, None]

    def call(i, val):
        a = list(args)
        a[i] = val
        return f(*a)

    assert call(2, 2) == wp.WP_ERR_ARG                  # layout outside the enum
    assert call(2, -1) == wp.WP_ERR_ARG
    assert call(1, None) == wp.WP_ERR_ARG               # K cache NULL
    assert call(15, ws - 1) == wp.WP_ERR_ARG            # workspace too small
    assert call(9, 80) == wp.WP_ERR_UNSUPPORTED         # d_h
    g = lib.wp_kcache_group_major
    assert g(None, FAKE, 1, 2, 100, 128, None) == wp.WP_ERR_ARG
    assert g(FAKE, FAKE, 1, 2, 100, 128, None) == wp.WP_ERR_ARG      # in place
    assert g(FAKE, FAKE + 8, 1, 2, 100, 128, None) == wp.WP_ERR_ARG  # misaligned
    assert g(FAKE, FAKE + 4096, 0, 2, 100, 128, None) == wp.WP_ERR_ARG
    assert g(FAKE, FAKE + 4096, 1, 2, 100, 80, None) == wp.WP_ERR_UNSUPPORTED


def test_decode_ex_per_head_channel_tables_checked(lib):
    """Exact rule with one channel row per query head: a NULL table, a
    negative cutoff and a table beyond the kernel parameter's 2048 entries
    are refused on the host, before any launch."""
    f = lib.wp_decode_ex
    ws = lib.wp_decode_workspace_bytes(2, 8, 128, 4096)

    def call(Hq, Hkv, cut):
        cp = None if cut is None else cut.ctypes.data_as(ctypes.c_void_p)
        return f(FAKE, FAKE, wp.KCACHE_ROWS, FAKE, FAKE, 4096, 2, Hq, Hkv, 128, wp.MODE_CHANNEL, cp, Hq,
                 wp.ROPE_HALF_SPLIT, ctypes.c_float(0.0), FAKE, None, FAKE, ws, None)

    assert call(8, 2, None) == wp.WP_ERR_ARG
    bad = np.full((8, 64), 100, dtype=np.int32)
    bad[5, 17] = -1
    assert call(8, 2, bad) == wp.WP_ERR_ARG
    big = np.full((64, 64), 100, dtype=np.int32)  # 64 heads x 64 channels = 4096 entries
    assert call(64, 8, big) == wp.WP_ERR_UNSUPPORTED


def test_decode_paged_rejects_bad_arguments(lib):
    f = lib.wp_decode_paged
    ws = lib.wp_decode_workspace_bytes(2, 8, 128, 64 * 64)
    # q, k_pages, k_layout, v_pages, n_pages, page_size, block_table, max_pages, lens, B, Hq, Hkv, d, cut, scale,
    # o, lse, ws, ws_bytes, stream
    args = [FAKE, FAKE, wp.KCACHE_ROWS, FAKE, 100, 64, FAKE, 64, FAKE, 2, 8, 2, 128, None, ctypes.c_float(0.0),
            FAKE, None, FAKE, ws, None]

    def call(i, val):
        a = list(args)
        a[i] = val
        return f(*a)

    assert call(6, None) == wp.WP_ERR_ARG               # block table NULL
    assert call(6, FAKE + 2) == wp.WP_ERR_ARG           # block table misaligned
    assert call(5, 8) == wp.WP_ERR_ARG                  # page size below 16
    assert call(5, 40) == wp.WP_ERR_ARG                 # page size not a multiple of 16
    assert call(4, 0) == wp.WP_ERR_ARG                  # empty pool
    assert call(7, 0) == wp.WP_ERR_ARG                  # no pages per sequence
    assert call(2, 5) == wp.WP_ERR_ARG                  # K layout
    assert call(18, ws - 1) == wp.WP_ERR_ARG            # workspace too small for max_pages * page_size keys
    assert call(7, 1 << 26) == wp.WP_ERR_UNSUPPORTED    # 2^32 keys per sequence


def test_decode_static_checks_pointers_before_sizes(lib):
    """A null or misaligned pointer is WP_ERR_ARG even for a batch too large
    for the fixed scratch; a well-formed oversized batch is WP_ERR_UNSUPPORTED.
    Neither reaches the GPU."""
    f = lib.wp_decode_static
    big = [FAKE, FAKE, FAKE, FAKE, 131072, 64, 64, 8, 128, None, ctypes.c_float(0.0), FAKE, None, None]
    assert lib.wp_decode_workspace_bytes(64, 64, 128, 131072) > wp.DECODE_STATIC_SCRATCH_BYTES

    def call(i, val):
        a = list(big)
        a[i] = val
        return f(*a)

    assert call(0, None) == wp.WP_ERR_ARG               # q NULL
    assert call(3, None) == wp.WP_ERR_ARG               # lens NULL
    assert call(11, FAKE + 8) == wp.WP_ERR_ARG          # o misaligned
    assert call(12, FAKE + 2) == wp.WP_ERR_ARG          # lse misaligned
    assert f(*big) == wp.WP_ERR_UNSUPPORTED


def test_rope_rejects_bad_arguments(lib):
    f = lib.wp_rope_apply
    assert f(None, FAKE, 1, 4, 2, 128, None, 0, 1e4, None, 1.0, 0, None) == wp.WP_ERR_ARG
    assert f(FAKE, FAKE + 64, 1, 4, 2, 128, None, 0, 1e4, None, 1.0, 0, None) == wp.WP_ERR_ARG  # partial overlap
    assert f(FAKE, FAKE, 1, 4, 2, 128, None, 0, 0.5, None, 1.0, 0, None) == wp.WP_ERR_ARG       # theta
    assert f(FAKE, FAKE, 1, 4, 2, 48, None, 0, 1e4, None, 1.0, 0, None) == wp.WP_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, 1, 4, 2, 128, None, 0, 1e4, None, 1.0, 3, None) == wp.WP_ERR_ARG       # layout
    # the paired half-split order permutes dims: never in place
    assert f(FAKE, FAKE, 1, 4, 2, 128, None, 0, 1e4, None, 1.0, wp.ROPE_HALF_SPLIT_PAIRED, None) == wp.WP_ERR_ARG


def test_status_strings(lib):
    for code in range(5):
        assert wp.wp_status_str(code)
    assert "unknown" in wp.wp_status_str(99)


def test_kcache_windowed_geometry_and_checks(lib):
    """Ring capacities round_up_16(W_g + 1), capped at round_up_16(Lmax);
    null or misaligned buffers and missing or negative tables are refused on
    the host."""
    def expect(Lmax, d, cut):
        lm = (Lmax + 15) // 16 * 16
        return 16 * sum(min((int(w) + 1 + 15) // 16 * 16, lm) for w in cut[: d // 16])
    for Lmax, d, cut in [(3000, 128, [5, 40, 300, 1100, 2000, 10 ** 6, 7, 1024]), (32768, 128, [160, 5063, 160114,
                         5063255] * 2), (1, 64, [0, 0, 0, 0]), (17, 64, [15, 16, 2 ** 31 - 1, 31])]:
        assert wp.wp_kcache_windowed_elems(Lmax, d, cut) == expect(Lmax, d, cut)
    P = ctypes.c_void_p
    cut = (ctypes.c_int32 * 8)(*([100] * 8))
    bad = (ctypes.c_int32 * 8)(*([100] * 7 + [-1]))
    assert lib.wp_kcache_windowed_elems(0, 128, cut) == 0
    assert lib.wp_kcache_windowed_elems(100, 128, None) == 0
    assert lib.wp_kcache_windowed_elems(100, 128, bad) == 0
    buf = ctypes.create_string_buffer(1 << 16)
    base = (ctypes.addressof(buf) + 255) & ~255
    assert lib.wp_kcache_windowed_from_rows(None, P(base), P(base + 4096), 1, 1, 16, 128, cut, None) == 1
    assert lib.wp_kcache_windowed_from_rows(P(base), P(base), P(base + 1), 1, 1, 16, 128, cut, None) == 1
    assert lib.wp_kcache_windowed_from_rows(P(base), P(base), P(base + 4096), 1, 1, 16, 128, None, None) == 1
    assert lib.wp_kcache_windowed_append(P(base), P(base + 2), P(base + 4096), 1, 1, 16, 128, cut, None) == 1
    assert lib.wp_kcache_windowed_append(P(base), P(base), P(base + 4096), 0, 1, 16, 128, cut, None) == 1
    assert lib.wp_kcache_windowed_from_rows(P(base), P(base), P(base + 4096), 1, 1, 16, 96, cut, None) == 2
