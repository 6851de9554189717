"""The seeded input recipe: deterministic per workload, the stated shapes,
distributions and length ranges, bf16-rounded values. Host only."""
import torch

import wp_synthetic as syn


def test_workloads_are_deterministic_and_shaped():
    w = syn.workload("tiny")
    a = syn.prefill_inputs(w)
    b = syn.prefill_inputs(w)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    q, k, v = a
    assert q.shape == (w.B, w.N, w.Hq, w.d) and k.shape == (w.B, w.N, w.Hkv, w.d) and v.shape == k.shape
    assert q.dtype == k.dtype == v.dtype == torch.bfloat16
    # another seed gives other values
    q2, _, _ = syn.prefill_inputs(w, seed=12345)
    assert not torch.equal(q, q2)


def test_values_are_standard_normal_rounded_to_bf16():
    w = syn.workload("tiny")
    q, k, v = syn.prefill_inputs(w)
    x = torch.cat([q.float().ravel(), k.float().ravel(), v.float().ravel()])
    assert abs(float(x.mean())) < 0.02 and abs(float(x.std()) - 1.0) < 0.02
    assert torch.equal(x.to(torch.bfloat16).float(), x)  # already bf16 values


def test_decode_lengths_in_range():
    w = syn.workload("decode_32k")
    q, kc, vc, lens = syn.decode_inputs(w, B=64, Lmax=4096, Lmin=2048)
    assert lens.dtype == torch.int32 and int(lens.min()) >= 2048 and int(lens.max()) <= 4096
    assert kc.shape == (64, w.Hkv, 4096, w.d) and q.shape == (64, w.Hq, w.d)


def test_sampled_rows_cover_the_last_row():
    w = syn.workload("long_32k")
    rb, rh, ri = syn.sample_rows(w, 8)
    assert int(ri.max()) == w.N - 1
    assert set(rh.tolist()) == set(range(w.Hq))
