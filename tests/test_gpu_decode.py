"""GPU parity of wp_decode (split-KV, grouped cutoffs) against the fp64
oracle, plus decode-vs-prefill consistency on the GPU."""
import numpy as np
import pytest
import torch

import oracle
import rope_period_truncated_b200 as wp
import wp_synthetic as syn
from parity import assert_attention_close, widen

pytestmark = pytest.mark.gpu


def _gpu_decode(q, kc, vc, lens, cut):
    o, lse = wp.wp_decode(q.cuda(), kc.cuda(), vc.cuda(), lens.cuda(), cut)
    torch.cuda.synchronize()
    assert wp.wp_device_status() == 0
    return o, lse


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (4, 4), (8, 4), (16, 2)])
@pytest.mark.parametrize("d", [64, 128])
def test_decode_small(Hq, Hkv, d):
    g = torch.Generator().manual_seed(21 + Hq + d)
    B, Lmax = 4, 3000
    lens = torch.tensor([1, 2999, 1500, 1025], dtype=torch.int32)
    q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, Hkv, Lmax, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, Hkv, Lmax, d, generator=g).to(torch.bfloat16)
    _, wg = oracle.cutoffs(d, 1e4, oracle.HALF_SPLIT)
    wg = np.minimum(wg, [5, 40, 300, 1100, 2000, 10 ** 6, 7, 1024][: d // 16]).astype(np.int32)
    o, lse = _gpu_decode(q, kc, vc, lens, wg)
    ro, rl = oracle.decode(widen(q), widen(kc), widen(vc), lens.numpy(), wg)
    assert_attention_close(o, lse, ro, rl, f"decode Hq={Hq} Hkv={Hkv} d={d}")


def test_decode_dense_and_zero_cutoffs():
    g = torch.Generator().manual_seed(3)
    B, Hq, Hkv, d, Lmax = 2, 8, 2, 128, 2100
    lens = torch.tensor([2100, 777], dtype=torch.int32)
    q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, Hkv, Lmax, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, Hkv, Lmax, d, generator=g).to(torch.bfloat16)
    for cut in [None, np.zeros(8, dtype=np.int32)]:
        o, lse = _gpu_decode(q, kc, vc, lens, cut)
        ocut = cut if cut is not None else np.full(8, 2 ** 31 - 1)
        ro, rl = oracle.decode(widen(q), widen(kc), widen(vc), lens.numpy(), ocut)
        assert_attention_close(o, lse, ro, rl, f"decode cut={'dense' if cut is None else 'zero'}")


def test_decode_large_logits():
    """Logits spanning hundreds of base-2 units (q and K scaled by 8, older
    keys scaled up to 3x more): within a split most exponentials underflow,
    and the splits' maxima differ by far more than fp32's range, so the
    combine's LSE merge carries the result. Lengths across several 1024-key
    splits with ragged ends."""
    g = torch.Generator().manual_seed(77)
    B, Hq, Hkv, d, Lmax = 3, 8, 2, 128, 3500
    lens = torch.tensor([3500, 2049, 700], dtype=torch.int32)
    ramp = (1.0 + 2.0 * torch.arange(Lmax - 1, -1, -1, dtype=torch.float32) / Lmax).view(1, 1, Lmax, 1)
    q = (8.0 * torch.randn(B, Hq, d, generator=g)).to(torch.bfloat16)
    kc = (8.0 * ramp * torch.randn(B, Hkv, Lmax, d, generator=g)).to(torch.bfloat16)
    vc = torch.randn(B, Hkv, Lmax, d, generator=g).to(torch.bfloat16)
    _, wg = oracle.cutoffs(d, 1e4, oracle.HALF_SPLIT)
    s2 = (widen(q)[0, 0] @ widen(kc)[0, 0].T) / np.sqrt(d) / np.log(2.0)
    assert s2.max() - s2.min() > 240  # the case is what it claims
    o, lse = _gpu_decode(q, kc, vc, lens, wg)
    ro, rl = oracle.decode(widen(q), widen(kc), widen(vc), lens.numpy(), wg)
    assert_attention_close(o, lse, ro, rl, "decode large logits")


def test_decode_workload_full():
    """16 sequences, H32/8, d128, lengths U[16384, 32768], theta 1e6 half-split:
    the query is rotated on the GPU at position len-1, every row checked."""
    w = syn.workload("decode_32k")
    q, kc, vc, lens = syn.decode_inputs(w)
    _, wg = oracle.cutoffs(w.d, w.theta, w.layout)
    pos = (lens - 1).to(torch.int32).reshape(w.B, 1)
    qr = wp.wp_rope_apply(q.cuda().reshape(w.B, 1, w.Hq, w.d), w.theta, w.layout, pos=pos.cuda())
    o, lse = wp.wp_decode(qr.reshape(w.B, w.Hq, w.d), kc.cuda(), vc.cuda(), lens.cuda(), wg)
    torch.cuda.synchronize()
    assert wp.wp_device_status() == 0
    qo = oracle.rope(widen(q).reshape(w.B, 1, w.Hq, w.d), w.theta, w.layout, pos=pos.numpy())
    qo = oracle.bf16_bits_to_f64(oracle.round_bf16_bits(qo)).reshape(w.B, w.Hq, w.d)
    ro, rl = oracle.decode(qo, widen(kc), widen(vc), lens.numpy(), wg)
    assert_attention_close(o, lse, ro, rl, "decode_32k")


def test_decode_matches_prefill_last_row():
    """Decode at length L equals row L-1 of the GPU prefill over the same keys."""
    g = torch.Generator().manual_seed(9)
    Hq, Hkv, d, L = 8, 2, 128, 1000
    q = torch.randn(1, L, Hq, d, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(1, L, Hkv, d, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(1, L, Hkv, d, generator=g).to(torch.bfloat16).cuda()
    _, wg = oracle.cutoffs(d, 1e6, oracle.HALF_SPLIT)
    po, pl = wp.wp_prefill(q, k, v, wg)
    kc = k.permute(0, 2, 1, 3).contiguous()
    vc = v.permute(0, 2, 1, 3).contiguous()
    do, dl = wp.wp_decode(q[:, L - 1].contiguous(), kc, vc, torch.tensor([L], dtype=torch.int32, device="cuda"), wg)
    torch.cuda.synchronize()
    assert (do.float() - po[:, L - 1].float()).abs().max().item() < 2e-2
    assert (dl - pl[:, :, L - 1]).abs().max().item() < 1e-3 * max(1.0, pl[:, :, L - 1].abs().max().item())


def test_decode_bad_length_gives_nan_rows():
    """A length outside 1..Lmax yields NaN rows for that sequence only."""
    B, Hq, Hkv, d, Lmax = 2, 4, 1, 64, 256
    q = torch.ones(B, Hq, d, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(B, Hkv, Lmax, d, dtype=torch.bfloat16, device="cuda")
    vc = torch.ones(B, Hkv, Lmax, d, dtype=torch.bfloat16, device="cuda")
    lens = torch.tensor([0, 100], dtype=torch.int32, device="cuda")
    o, lse = wp.wp_decode(q, kc, vc, lens, None)
    torch.cuda.synchronize()
    assert torch.isnan(o[0].float()).all() and torch.isnan(lse[0]).all()
    assert torch.allclose(o[1].float(), torch.ones_like(o[1].float()))


def test_kcache_group_major_layout():
    """wp_kcache_group_major is the permutation [B,Hkv,L,G,16] -> [B,Hkv,G,L,16]."""
    g = torch.Generator().manual_seed(11)
    for d in (64, 128):
        kc = torch.randn(3, 2, 1000, d, generator=g).to(torch.bfloat16).cuda()
        gm = wp.wp_kcache_group_major(kc)
        torch.cuda.synchronize()
        want = kc.reshape(3, 2, 1000, d // 16, 16).permute(0, 1, 3, 2, 4).contiguous()
        assert torch.equal(gm, want)


@pytest.mark.parametrize("d", [64, 128])
def test_decode_group_major_kcache(d):
    """The group-major K cache gives results bit-identical to the row layout,
    and both match the oracle (ragged lengths, boundary cutoffs)."""
    g = torch.Generator().manual_seed(31 + d)
    B, Hq, Hkv, Lmax = 4, 8, 2, 3000
    lens = torch.tensor([1, 2999, 1500, 1025], dtype=torch.int32)
    q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, Hkv, Lmax, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, Hkv, Lmax, d, generator=g).to(torch.bfloat16)
    _, wg = oracle.cutoffs(d, 1e4, oracle.HALF_SPLIT)
    wg = np.minimum(wg, [5, 40, 300, 1100, 2000, 10 ** 6, 7, 1024][: d // 16]).astype(np.int32)
    o_rows, lse_rows = _gpu_decode(q, kc, vc, lens, wg)
    kgm = wp.wp_kcache_group_major(kc.cuda())
    o_gm, lse_gm = wp.wp_decode(q.cuda(), kgm, vc.cuda(), lens.cuda(), wg)
    torch.cuda.synchronize()
    assert wp.wp_device_status() == 0
    assert torch.equal(o_gm, o_rows) and torch.equal(lse_gm, lse_rows)
    ro, rl = oracle.decode(widen(q), widen(kc), widen(vc), lens.numpy(), wg)
    assert_attention_close(o_gm, lse_gm, ro, rl, f"decode group-major d={d}")


@pytest.mark.parametrize("d", [64, 128])
def test_decode_windowed_kcache(d):
    """Evicting every group's out-of-window keys changes nothing: the windowed
    K cache (per-group rings of round_up_16(W_g + 1) keys, wrapping many times
    for the small cutoffs here) gives results bit-identical to the full cache
    and matches the oracle; appending each sequence's last key to a cache
    built for one key less gives the same cache, slot for slot."""
    g = torch.Generator().manual_seed(41 + d)
    B, Hq, Hkv, Lmax = 4, 8, 2, 3000
    lens = torch.tensor([1, 2999, 1500, 1025], dtype=torch.int32)
    q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, Hkv, Lmax, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, Hkv, Lmax, d, generator=g).to(torch.bfloat16)
    wg = np.array([5, 40, 300, 1100, 2000, 10 ** 6, 7, 1024][: d // 16], dtype=np.int32)
    o_rows, lse_rows = _gpu_decode(q, kc, vc, lens, wg)
    kw = wp.wp_kcache_windowed(kc.cuda(), lens.cuda(), wg)
    caps = [min((int(w) + 1 + 15) // 16 * 16, (Lmax + 15) // 16 * 16) for w in wg]
    assert kw.shape == (B, Hkv, 16 * sum(caps)) and kw.shape[2] < Lmax * d
    o_w, lse_w = wp.wp_decode(q.cuda(), kw, vc.cuda(), lens.cuda(), wg)
    torch.cuda.synchronize()
    assert wp.wp_device_status() == 0
    assert torch.equal(o_w, o_rows) and torch.equal(lse_w, lse_rows)
    ro, rl = oracle.decode(widen(q), widen(kc), widen(vc), lens.numpy(), wg)
    assert_attention_close(o_w, lse_w, ro, rl, f"decode windowed d={d}")
    # one decode step: the cache for len - 1 keys plus the key at len - 1
    kw_prev = wp.wp_kcache_windowed(kc.cuda(), (lens - 1).cuda(), wg)
    k_new = torch.stack([kc[b, :, int(lens[b]) - 1, :] for b in range(B)]).contiguous()
    wp.wp_kcache_windowed_append(k_new.cuda(), (lens - 1).cuda(), kw_prev, Lmax, wg)
    torch.cuda.synchronize()
    assert torch.equal(kw_prev, kw)


def test_decode_group_major_workload():
    """The 32K decode workload with a group-major K cache: every row checked
    against the oracle."""
    w = syn.workload("decode_32k")
    q, kc, vc, lens = syn.decode_inputs(w)
    _, wg = oracle.cutoffs(w.d, w.theta, w.layout)
    pos = (lens - 1).to(torch.int32).reshape(w.B, 1)
    qr = wp.wp_rope_apply(q.cuda().reshape(w.B, 1, w.Hq, w.d), w.theta, w.layout, pos=pos.cuda())
    kgm = wp.wp_kcache_group_major(kc.cuda())
    o, lse = wp.wp_decode(qr.reshape(w.B, w.Hq, w.d), kgm, vc.cuda(), lens.cuda(), wg)
    torch.cuda.synchronize()
    assert wp.wp_device_status() == 0
    qo = oracle.rope(widen(q).reshape(w.B, 1, w.Hq, w.d), w.theta, w.layout, pos=pos.numpy())
    qo = oracle.bf16_bits_to_f64(oracle.round_bf16_bits(qo)).reshape(w.B, w.Hq, w.d)
    ro, rl = oracle.decode(qo, widen(kc), widen(vc), lens.numpy(), wg)
    assert_attention_close(o, lse, ro, rl, "decode_32k group-major")


def _paged(kc, vc, P, extra, seed):
    """Contiguous caches [B,Hkv,L,d] (L a multiple of P) -> shuffled page pools
    [n_pages,Hkv,P,d] and the block table [B, L/P]."""
    B, Hkv, L, d = kc.shape
    mp = L // P

    def pool_of(x):
        pages = x.reshape(B, Hkv, mp, P, d).permute(0, 2, 1, 3, 4).reshape(B * mp, Hkv, P, d)
        return pages

    g = torch.Generator().manual_seed(seed)
    n_pages = B * mp + extra
    perm = torch.randperm(n_pages, generator=g)[: B * mp]
    kp = torch.zeros((n_pages, Hkv, P, d), dtype=kc.dtype)
    vp = torch.zeros((n_pages, Hkv, P, d), dtype=vc.dtype)
    kp[perm] = pool_of(kc)
    vp[perm] = pool_of(vc)
    table = perm.to(torch.int32).reshape(B, mp)
    return kp, vp, table


@pytest.mark.parametrize("P", [16, 64, 256])
@pytest.mark.parametrize("group_major", [False, True])
def test_decode_paged_matches_contiguous(P, group_major):
    """A paged cache (shuffled pages in a larger pool) gives results
    bit-identical to the same keys stored contiguously, in both K layouts."""
    g = torch.Generator().manual_seed(61 + P)
    B, Hq, Hkv, d, L = 3, 8, 2, 128, 3072
    lens = torch.tensor([1, 3072, 1700], dtype=torch.int32)
    q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, Hkv, L, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, Hkv, L, d, generator=g).to(torch.bfloat16)
    _, wg = oracle.cutoffs(d, 1e4, oracle.HALF_SPLIT)
    wg = np.minimum(wg, [5, 40, 300, 1100, 2000, 10 ** 6, 7, 1024]).astype(np.int32)
    kp, vp, table = _paged(kc, vc, P, extra=5, seed=P)
    kcd, kpd = kc.cuda(), kp.cuda()
    if group_major:
        kcd = wp.wp_kcache_group_major(kcd)
        n = kp.shape[0]
        kpd = kpd.reshape(n, Hkv, P, d // 16, 16).permute(0, 1, 3, 2, 4).contiguous()
    o_ref, l_ref = wp.wp_decode(q.cuda(), kcd, vc.cuda(), lens.cuda(), wg)
    o, lse = wp.wp_decode_paged(q.cuda(), kpd, vp.cuda(), table.cuda(), lens.cuda(), wg)
    torch.cuda.synchronize()
    assert wp.wp_device_status() == 0
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
    ro, rl = oracle.decode(widen(q), widen(kc), widen(vc), lens.numpy(), wg)
    assert_attention_close(o, lse, ro, rl, f"paged P={P} gm={group_major}")


def test_decode_paged_bad_page_gives_nan_rows():
    """A block-table entry outside the pool poisons only its own sequence."""
    g = torch.Generator().manual_seed(9)
    B, Hq, Hkv, d, L, P = 2, 4, 2, 64, 512, 64
    lens = torch.tensor([512, 300], dtype=torch.int32)
    q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, Hkv, L, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, Hkv, L, d, generator=g).to(torch.bfloat16)
    kp, vp, table = _paged(kc, vc, P, extra=0, seed=1)
    table[1, 2] = kp.shape[0] + 7  # a page of sequence 1 that does not exist
    o, lse = wp.wp_decode_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), lens.cuda(), None)
    torch.cuda.synchronize()
    assert wp.wp_device_status() == 0
    o = o.float().cpu()
    assert torch.isnan(o[1]).all()
    ro, rl = oracle.decode(widen(q[:1]), widen(kc[:1]), widen(vc[:1]), lens[:1].numpy(), np.full(d // 16, 2 ** 31 - 1))
    assert_attention_close(o[:1].to(torch.bfloat16), lse[:1], ro, rl, "paged, sequence with valid pages")


def _decode_inputs(seed, B, Hq, Hkv, d, Lmax):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, Hkv, Lmax, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, Hkv, Lmax, d, generator=g).to(torch.bfloat16)
    return q, kc, vc


@pytest.mark.parametrize("group_major", [False, True])
@pytest.mark.parametrize("Hq,Hkv,d", [(8, 2, 128), (4, 4, 64), (16, 2, 128)])
def test_decode_per_head_tables(Hq, Hkv, d, group_major):
    """One cutoff row per query head (wp_decode_ex, grouped): the K loads
    cover the union of the heads' windows and each head keeps a group's
    product only inside its own window. Oracle: one head at a time."""
    B, Lmax = 4, 3000
    lens = torch.tensor([1, 2999, 1500, 1025], dtype=torch.int32)
    q, kc, vc = _decode_inputs(61 + Hq + d, B, Hq, Hkv, d, Lmax)
    rng = np.random.default_rng(Hq * 7 + d)
    G = d // 16
    cut = rng.integers(0, 2500, size=(Hq, G)).astype(np.int32)
    cut[0] = 2 ** 31 - 1  # a dense head next to pruned ones
    kcd = wp.wp_kcache_group_major(kc.cuda()) if group_major else kc.cuda()
    o, lse = wp.wp_decode(q.cuda(), kcd, vc.cuda(), lens.cuda(), cut)
    torch.cuda.synchronize()
    assert wp.wp_device_status() == 0
    ro = np.zeros((B, Hq, d))
    rl = np.zeros((B, Hq))
    for h in range(Hq):
        hk = h // (Hq // Hkv)
        a, b_ = oracle.decode(widen(q[:, h:h + 1]), widen(kc[:, hk:hk + 1]), widen(vc[:, hk:hk + 1]), lens.numpy(),
                              cut[h])
        ro[:, h], rl[:, h] = a[:, 0], b_[:, 0]
    assert_attention_close(o, lse, ro, rl, f"per-head decode Hq={Hq} d={d} gm={group_major}")


@pytest.mark.parametrize("layout", [wp.ROPE_INTERLEAVED, wp.ROPE_HALF_SPLIT])
@pytest.mark.parametrize("group_major", [False, True])
@pytest.mark.parametrize("table", ["wave", "small"])
def test_decode_exact_channel_mode(layout, group_major, table):
    """Exact per-channel rule in decode (wp_decode_ex, channel mode) against
    the oracle's channel-mode row len-1 over the cached keys."""
    B, Hq, Hkv, d, Lmax = 3, 8, 2, 128, 2600
    lens = torch.tensor([2600, 700, 1], dtype=torch.int32)
    q, kc, vc = _decode_inputs(71 + layout, B, Hq, Hkv, d, Lmax)
    if table == "wave":
        wc, _ = oracle.cutoffs(d, 1e4, layout)
    else:
        wc = np.random.default_rng(5).integers(0, 600, size=d // 2).astype(np.int32)
    kcd = wp.wp_kcache_group_major(kc.cuda()) if group_major else kc.cuda()
    o, lse = wp.wp_decode(q.cuda(), kcd, vc.cuda(), lens.cuda(), wc, mode=wp.MODE_CHANNEL, layout=layout)
    torch.cuda.synchronize()
    assert wp.wp_device_status() == 0
    # oracle: row len-1 of channel-mode prefill over the cached keys ([B, L, Hkv, d] order)
    rb = np.repeat(np.arange(B), Hq)
    rh = np.tile(np.arange(Hq), B)
    ri = (lens.numpy().astype(np.int64) - 1)[rb]
    ro, rl = oracle.attention_rows(widen(q).reshape(B * Hq, d), (rb, rh, ri), widen(kc).transpose(0, 2, 1, 3),
                                   widen(vc).transpose(0, 2, 1, 3), Hq, wc, oracle.MODE_CHANNEL, layout)
    assert_attention_close(o, lse, ro.reshape(B, Hq, d), rl.reshape(B, Hq), f"exact decode layout={layout}")


@pytest.mark.parametrize("layout", [wp.ROPE_INTERLEAVED, wp.ROPE_HALF_SPLIT])
@pytest.mark.parametrize("group_major", [False, True])
@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (8, 1), (4, 4)])
def test_decode_exact_per_head_tables(layout, group_major, Hq, Hkv):
    """Exact per-channel rule with one channel row per query head
    (wp_decode_ex, channel mode, cut_rows = H_q): the heads of a KV head
    share its K loads, each head's product takes K masked by its own row.
    Oracle: channel-mode row len-1 one head at a time."""
    B, d, Lmax = 3, 128, 2600
    lens = torch.tensor([2600, 700, 1], dtype=torch.int32)
    q, kc, vc = _decode_inputs(91 + layout + Hq + Hkv, B, Hq, Hkv, d, Lmax)
    rng = np.random.default_rng(Hq * 3 + Hkv + layout)
    cut = rng.integers(0, 2000, size=(Hq, d // 2)).astype(np.int32)
    cut[1] = 2 ** 31 - 1  # a dense head next to pruned ones
    kcd = wp.wp_kcache_group_major(kc.cuda()) if group_major else kc.cuda()
    o, lse = wp.wp_decode(q.cuda(), kcd, vc.cuda(), lens.cuda(), cut, mode=wp.MODE_CHANNEL, layout=layout)
    torch.cuda.synchronize()
    assert wp.wp_device_status() == 0
    kr, vr = widen(kc).transpose(0, 2, 1, 3), widen(vc).transpose(0, 2, 1, 3)
    ri = lens.numpy().astype(np.int64) - 1
    ro = np.zeros((B, Hq, d))
    rl = np.zeros((B, Hq))
    for h in range(Hq):
        a, b_ = oracle.attention_rows(widen(q)[:, h], (np.arange(B), np.full(B, h), ri), kr, vr, Hq, cut[h],
                                      oracle.MODE_CHANNEL, layout)
        ro[:, h], rl[:, h] = a.reshape(B, d), b_.reshape(B)
    assert_attention_close(o, lse, ro, rl, f"exact per-head decode Hq={Hq} Hkv={Hkv} gm={group_major}")
