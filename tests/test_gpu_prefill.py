"""GPU parity of wp_prefill (grouped tcgen05 path and exact channel path)
against the fp64 oracle, on the same seeded inputs.

Small cases and the Qwen3-shaped 4K workload run the oracle on every row
(several 128-row tiles plus ragged tails, multiple boundary cutoffs per tile,
all-masked and dense tables); the 32K and 128K workloads are checked on
sampled rows, through the same launch
(rope of Q and K, then prefill) that the bench times."""
import numpy as np
import pytest
import torch

import oracle
import rope_period_truncated_b200 as wp
import wp_synthetic as syn
from parity import assert_attention_close, widen

pytestmark = pytest.mark.gpu


def _oracle_rotated(x_bf16, theta, layout, scale_all=1.0):
    """The oracle's own rotation of the bf16 input, rounded to bf16, widened."""
    r = oracle.rope(widen(x_bf16), theta, layout, scale_all=scale_all)
    return oracle.bf16_bits_to_f64(oracle.round_bf16_bits(r))


def _gpu_path(q, k, v, theta, layout, cut, mode, scale_all=1.0, rope=True):
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    if rope:
        qg = wp.wp_rope_apply(qg, theta, layout, scale_all=scale_all)
        kg = wp.wp_rope_apply(kg, theta, layout, scale_all=scale_all)
    o, lse = wp.wp_prefill(qg, kg, vg, cut, mode, layout)
    torch.cuda.synchronize()
    assert wp.wp_device_status() == 0
    return o, lse


@pytest.mark.parametrize("mode", [wp.MODE_GROUPED, wp.MODE_CHANNEL])
def test_tiny_workload(mode):
    """Tiny workload: B1 H2/2 N256 d64 theta 1e4, interleaved; both modes."""
    w = syn.workload("tiny")
    q, k, v = syn.prefill_inputs(w)
    wc, wg = oracle.cutoffs(w.d, w.theta, w.layout)
    cut = wg if mode == wp.MODE_GROUPED else wc
    o, lse = _gpu_path(q, k, v, w.theta, w.layout, cut, mode)
    qr, kr = _oracle_rotated(q, w.theta, w.layout), _oracle_rotated(k, w.theta, w.layout)
    ro, rl = oracle.attention(qr, kr, widen(v), cut, mode, w.layout)
    assert_attention_close(o, lse, ro, rl, f"tiny mode={mode}")


def _cut_table(kind, d, theta, layout, mode):
    G, C = d // 16, d // 2
    n = G if mode == wp.MODE_GROUPED else C
    if kind == "wave":
        wc, wg = oracle.cutoffs(d, theta, layout)
        return wg if mode == wp.MODE_GROUPED else wc
    if kind == "dense":
        return None
    if kind == "zero":
        return np.zeros(n, dtype=np.int32)
    if kind == "mixed":  # several distinct cutoffs inside one 128x128 tile
        base = np.array([0, 3, 130, 129, 50, 200, 255, 1000], dtype=np.int32)
        return np.resize(base, n)
    if kind == "alternate":  # every group holds dropped and kept channels at every distance
        return np.where(np.arange(n) % 2 == 0, 0, 2 ** 30).astype(np.int32)
    if kind == "spread":  # a distinct cutoff per entry, many inside one 64-key sub-tile
        return ((np.arange(n) * 37) % 301).astype(np.int32)
    raise ValueError(kind)


SMALL = [
    # N, d, Hq, Hkv, theta, layout, kind
    (1, 128, 2, 1, 1e6, wp.ROPE_HALF_SPLIT, "wave"),
    (127, 64, 2, 2, 1e4, wp.ROPE_INTERLEAVED, "wave"),
    (129, 128, 4, 2, 1e4, wp.ROPE_HALF_SPLIT, "wave"),
    (300, 128, 4, 1, 1e6, wp.ROPE_INTERLEAVED, "wave"),   # 28 and 160 boundary in one tile
    (513, 128, 8, 2, 1e4, wp.ROPE_HALF_SPLIT, "wave"),
    (640, 128, 4, 4, 1e6, wp.ROPE_HALF_SPLIT, "mixed"),
    (384, 64, 4, 2, 1e4, wp.ROPE_INTERLEAVED, "mixed"),
    (300, 128, 2, 2, 1e6, wp.ROPE_HALF_SPLIT, "zero"),
    (300, 128, 2, 2, 1e6, wp.ROPE_HALF_SPLIT, "dense"),
    (190, 128, 6, 2, 1e4, wp.ROPE_HALF_SPLIT, "wave"),    # 3 query heads per KV head: one head per CTA;
                                                          # last tile of 62 rows (< one 64-key half)
    (200, 64, 6, 3, 1e4, wp.ROPE_INTERLEAVED, "mixed"),   # 2 per KV head; last tile of 72 rows
    (400, 128, 2, 1, 1e4, wp.ROPE_INTERLEAVED, "alternate"),  # 8 partially kept groups per sub-tile
    (400, 128, 2, 1, 1e4, wp.ROPE_HALF_SPLIT, "alternate"),
    (333, 128, 2, 2, 1e6, wp.ROPE_HALF_SPLIT, "spread"),
    (333, 64, 4, 2, 1e4, wp.ROPE_INTERLEAVED, "spread"),
]


@pytest.mark.parametrize("N,d,Hq,Hkv,theta,layout,kind", SMALL)
@pytest.mark.parametrize("mode", [wp.MODE_GROUPED, wp.MODE_CHANNEL])
def test_small_full_rows(N, d, Hq, Hkv, theta, layout, kind, mode):
    g = torch.Generator().manual_seed(100 + N + d)
    q = torch.randn(2, N, Hq, d, generator=g).to(torch.bfloat16)
    k = torch.randn(2, N, Hkv, d, generator=g).to(torch.bfloat16)
    v = torch.randn(2, N, Hkv, d, generator=g).to(torch.bfloat16)
    cut = _cut_table(kind, d, theta, layout, mode)
    # prefill alone on the drawn values (treated as already rotated)
    o, lse = _gpu_path(q, k, v, theta, layout, cut, mode, rope=False)
    ocut = cut if cut is not None else np.full(d // 16 if mode == wp.MODE_GROUPED else d // 2, 2 ** 31 - 1)
    ro, rl = oracle.attention(widen(q), widen(k), widen(v), ocut, mode, layout)
    assert_attention_close(o, lse, ro, rl, f"N={N} d={d} {kind} mode={mode}")


@pytest.mark.parametrize("mode", [wp.MODE_GROUPED, wp.MODE_CHANNEL])
def test_large_logits(mode):
    """Logits spanning hundreds of base-2 units (Q and K scaled by 8, keys
    further from the diagonal scaled up to 3x more): most exponentials fall
    below the polynomial exp2's clamp at 2^-120, and row maxima keep growing
    past the 2^8 rescale threshold as the kernel walks the key tiles back from
    the diagonal. 700 rows: several tiles and a ragged tail."""
    N, d, Hq, Hkv, theta, layout = 700, 128, 4, 2, 1e4, wp.ROPE_HALF_SPLIT
    g = torch.Generator().manual_seed(4242)
    ramp = (1.0 + 2.0 * torch.arange(N - 1, -1, -1, dtype=torch.float32) / N).view(1, N, 1, 1)
    q = (8.0 * torch.randn(1, N, Hq, d, generator=g)).to(torch.bfloat16)
    k = (8.0 * ramp * torch.randn(1, N, Hkv, d, generator=g)).to(torch.bfloat16)
    v = torch.randn(1, N, Hkv, d, generator=g).to(torch.bfloat16)
    cut = _cut_table("wave", d, theta, layout, mode)
    o, lse = _gpu_path(q, k, v, theta, layout, cut, mode, rope=False)
    ro, rl = oracle.attention(widen(q), widen(k), widen(v), cut, mode, layout)
    # the case is what it claims: the last row's unmasked logits span far more
    # than 120 base-2 units
    s2 = (widen(q)[0, N - 1, 0] @ widen(k)[0, :, 0].T) / np.sqrt(d) / np.log(2.0)
    assert s2.max() - s2.min() > 240
    assert_attention_close(o, lse, ro, rl, f"large logits mode={mode}")


def _sampled_check(name, per_head, mode=wp.MODE_GROUPED):
    w = syn.workload(name)
    q, k, v = syn.prefill_inputs(w)
    wc, wg = oracle.cutoffs(w.d, w.theta, w.layout, scale_all=w.scale_all)
    cut = wg if mode == wp.MODE_GROUPED else wc
    o, lse = _gpu_path(q, k, v, w.theta, w.layout, cut, mode, scale_all=w.scale_all)
    rb, rh, ri = syn.sample_rows(w, per_head)
    # oracle: its own rotation of every key and of the sampled query rows
    kr = _oracle_rotated(k, w.theta, w.layout, w.scale_all)
    qrows = q[rb, ri, rh].unsqueeze(0).unsqueeze(2)            # [1, R, 1, d]
    qrot = oracle.rope(widen(qrows), w.theta, w.layout, pos=ri.numpy().reshape(1, -1), scale_all=w.scale_all)
    qrot = oracle.bf16_bits_to_f64(oracle.round_bf16_bits(qrot))[0, :, 0]
    ro, rl = oracle.attention_rows(qrot, (rb.numpy(), rh.numpy(), ri.numpy()), kr, widen(v), w.Hq, cut,
                                   mode, w.layout)
    og = o[rb.cuda(), ri.cuda(), rh.cuda()]
    lg = lse[rb.cuda(), rh.cuda(), ri.cuda()]
    return assert_attention_close(og, lg, ro, rl, f"{name} mode={mode}")


@pytest.mark.parametrize("mode", [wp.MODE_GROUPED, wp.MODE_CHANNEL])
def test_qwen3_shaped_every_row(mode):
    """B2 H32/8 N4096 d128 theta 1e6 half-split, per-dim Q/K scales: every
    row of every head (262,144 rows) against the oracle, through the same
    rope + prefill launches the bench times; grouped and exact rule."""
    w = syn.workload("qwen3_8b_4k")
    q, k, v = syn.prefill_inputs(w)
    wc, wg = oracle.cutoffs(w.d, w.theta, w.layout, scale_all=w.scale_all)
    cut = wg if mode == wp.MODE_GROUPED else wc
    o, lse = _gpu_path(q, k, v, w.theta, w.layout, cut, mode, scale_all=w.scale_all)
    qr = _oracle_rotated(q, w.theta, w.layout, w.scale_all)
    kr = _oracle_rotated(k, w.theta, w.layout, w.scale_all)
    ro, rl = oracle.attention(qr, kr, widen(v), cut, mode, w.layout)
    assert_attention_close(o, lse, ro, rl, f"qwen3_8b_4k every row mode={mode}")


@pytest.mark.parametrize("mode", [wp.MODE_GROUPED, wp.MODE_CHANNEL])
def test_long_32k_sampled_rows(mode):
    """B1 H32/8 N32768: 256 sampled rows per head; grouped and exact rule."""
    _sampled_check("long_32k", 256, mode)


def test_scaled_128k_sampled_rows():
    """B1 H32/8 N131072, every f_c divided by 4: 128 sampled rows per head."""
    _sampled_check("scaled_128k", 128)


def test_dense_is_cutoff_infinity():
    """cut=None (dense comparison path) equals an all-WP_CUTOFF_INF table bit for bit."""
    g = torch.Generator().manual_seed(5)
    q = torch.randn(1, 700, 4, 128, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(1, 700, 2, 128, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(1, 700, 2, 128, generator=g).to(torch.bfloat16).cuda()
    o1, l1 = wp.wp_prefill(q, k, v, None)
    o2, l2 = wp.wp_prefill(q, k, v, np.full(8, 2 ** 31 - 1, dtype=np.int32))
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def _oracle_per_head(q, k, v, cut_rows, mode, layout):
    """The oracle one query head at a time, each with its own cutoff row.
    q [B,N,Hq,d], k/v [B,N,Hkv,d] (fp64 numpy); returns (o, lse) like attention."""
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    o = np.empty_like(q)
    lse = np.empty((B, Hq, N))
    for h in range(Hq):
        hk = h // (Hq // Hkv)
        oh, lh = oracle.attention(q[:, :, h:h + 1], k[:, :, hk:hk + 1], v[:, :, hk:hk + 1], cut_rows[h], mode,
                                  layout)
        o[:, :, h:h + 1] = oh
        lse[:, h] = lh[:, 0]
    return o, lse


def _per_head_table(Hq, d, theta, layout, mode, seed):
    """Distinct cutoff rows per query head: the pages' table at several
    period multiples alpha, and small random tables that put several
    boundary cutoffs into one tile."""
    rng = np.random.default_rng(seed)
    n = d // 16 if mode == wp.MODE_GROUPED else d // 2
    rows = []
    for h in range(Hq):
        if h % 3 == 2:
            rows.append(rng.integers(0, 400, size=n).astype(np.int32))
        else:
            wc, wg = oracle.cutoffs(d, theta, layout, alpha=[2.0, 0.5, 8.0, 1.0][h % 4])
            rows.append(wg if mode == wp.MODE_GROUPED else wc)
    return np.stack(rows)


@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (6, 2), (4, 4)])
@pytest.mark.parametrize("mode", [wp.MODE_GROUPED, wp.MODE_CHANNEL])
def test_per_head_cutoff_tables(Hq, Hkv, mode):
    """One cutoff row per query head ([H_q][G] or [H_q][C]); the two heads of
    a GQA pair (or a single head when H_q/H_kv is odd) share K loads."""
    N, d, theta, layout = 400, 128, 1e4, wp.ROPE_HALF_SPLIT
    g = torch.Generator().manual_seed(200 + Hq + Hkv)
    q = torch.randn(2, N, Hq, d, generator=g).to(torch.bfloat16)
    k = torch.randn(2, N, Hkv, d, generator=g).to(torch.bfloat16)
    v = torch.randn(2, N, Hkv, d, generator=g).to(torch.bfloat16)
    cut = _per_head_table(Hq, d, theta, layout, mode, seed=Hq)
    o, lse = wp.wp_prefill(q.cuda(), k.cuda(), v.cuda(), cut, mode, layout)
    torch.cuda.synchronize()
    assert wp.wp_device_status() == 0
    ro, rl = _oracle_per_head(widen(q), widen(k), widen(v), cut, mode, layout)
    assert_attention_close(o, lse, ro, rl, f"per-head Hq={Hq} Hkv={Hkv} mode={mode}")


VARLEN = [
    # lengths, d, Hq, Hkv, layout
    ([1, 127, 128, 129, 300, 513], 128, 4, 2, wp.ROPE_HALF_SPLIT),
    ([200, 64, 1, 257], 64, 6, 2, wp.ROPE_INTERLEAVED),
]


@pytest.mark.parametrize("lens,d,Hq,Hkv,layout", VARLEN)
@pytest.mark.parametrize("mode", [wp.MODE_GROUPED, wp.MODE_CHANNEL])
@pytest.mark.parametrize("per_head", [False, True])
def test_packed_batch_of_ragged_sequences(lens, d, Hq, Hkv, layout, mode, per_head):
    """Packed batch (cu_seqlens) of sequences of different lengths, none or
    some multiples of the 128-row tile; positions restart in every sequence.
    Every row of every sequence against the oracle run on that sequence."""
    theta = 1e4
    T = sum(lens)
    g = torch.Generator().manual_seed(300 + T + d)
    q = torch.randn(T, Hq, d, generator=g).to(torch.bfloat16)
    k = torch.randn(T, Hkv, d, generator=g).to(torch.bfloat16)
    v = torch.randn(T, Hkv, d, generator=g).to(torch.bfloat16)
    if per_head:
        cut = _per_head_table(Hq, d, theta, layout, mode, seed=T)
    else:
        wc, wg = oracle.cutoffs(d, theta, layout)
        cut = wg if mode == wp.MODE_GROUPED else wc
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    o, lse = wp.wp_prefill(q.cuda(), k.cuda(), v.cuda(), cut, mode, layout, cu_seqlens=cu.cuda(),
                           max_seqlen=max(lens))
    torch.cuda.synchronize()
    assert wp.wp_device_status() == 0
    assert tuple(o.shape) == (T, Hq, d) and tuple(lse.shape) == (Hq, T)
    rows = cut if per_head else np.stack([cut] * Hq)
    for b, (s0, s1) in enumerate(zip(cu[:-1].tolist(), cu[1:].tolist())):
        qs, ks, vs = (widen(t[s0:s1]).reshape(1, s1 - s0, -1, d) for t in (q, k, v))
        ro, rl = _oracle_per_head(qs, ks, vs, rows, mode, layout)
        assert_attention_close(o[s0:s1].unsqueeze(0), lse[:, s0:s1].unsqueeze(0), ro, rl,
                               f"seq {b} len {s1 - s0} mode={mode} per_head={per_head}")


def test_packed_batch_of_equal_lengths_is_the_uniform_batch():
    """A packed batch whose sequences all have length N gives the uniform
    batch's results: only the tile coordinates differ, and the rounding of
    the diagonal tile's exponentials (a packed batch takes them all on MUFU,
    so that masked keys of the next sequence weigh exactly 0). A misplaced
    row or tile would differ by O(1)."""
    B, N, Hq, Hkv, d = 3, 333, 4, 2, 128
    g = torch.Generator().manual_seed(17)
    q = torch.randn(B, N, Hq, d, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(B, N, Hkv, d, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(B, N, Hkv, d, generator=g).to(torch.bfloat16).cuda()
    _, wg = oracle.cutoffs(d, 1e4, oracle.HALF_SPLIT)
    o1, l1 = wp.wp_prefill(q, k, v, wg)
    cu = torch.arange(0, B * N + 1, N, dtype=torch.int32, device="cuda")
    o2, l2 = wp.wp_prefill(q.reshape(B * N, Hq, d), k.reshape(B * N, Hkv, d), v.reshape(B * N, Hkv, d), wg,
                           cu_seqlens=cu, max_seqlen=N)
    torch.cuda.synchronize()
    assert (o1.reshape(B * N, Hq, d).float() - o2.float()).abs().max().item() <= 1e-2
    assert (l1.permute(1, 0, 2).reshape(Hq, B * N) - l2).abs().max().item() <= 1e-4


@pytest.mark.parametrize("mode", [wp.MODE_GROUPED, wp.MODE_CHANNEL])
def test_packed_batch_bad_offsets_are_reported(mode):
    """Offsets that run backwards are not followed: the kernel records
    WP_ERR_ARG in the status word (read and cleared by wp_device_status),
    and a later correct call runs normally."""
    T, Hq, Hkv, d = 400, 2, 2, 128
    q = torch.randn(T, Hq, d, device="cuda").to(torch.bfloat16)
    k = torch.randn(T, Hkv, d, device="cuda").to(torch.bfloat16)
    cu_bad = torch.tensor([0, 300, 100, 400], dtype=torch.int32, device="cuda")
    wp.wp_prefill(q, k, k, None, mode, cu_seqlens=cu_bad, max_seqlen=300)
    assert wp.wp_device_status() == wp.WP_ERR_ARG
    cu = torch.tensor([0, 100, 400], dtype=torch.int32, device="cuda")
    o, lse = wp.wp_prefill(q, k, k, None, mode, cu_seqlens=cu, max_seqlen=300)
    assert wp.wp_device_status() == wp.WP_OK
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
