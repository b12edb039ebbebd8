"""The seeded input recipe: deterministic, right shapes/dtypes, heavy keys where asked."""
import math

import torch

import synthetic


def test_draw_is_deterministic_and_shaped():
    w = synthetic.custom("t", "bf16", 2, 4, 2, 64, 16, 4, True, "striped", 7)
    a = synthetic.make_inputs(w, "cpu")
    b = synthetic.make_inputs(w, "cpu")
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    q, k, v = a
    assert q.shape == (2, 4, 64, 16) and k.shape == (2, 2, 64, 16) and v.shape == k.shape
    assert q.dtype == torch.bfloat16 and q.is_contiguous()
    # the recipe: fp32 randn in the order q, k, v then round to the dtype
    g = torch.Generator().manual_seed(7)
    q32 = torch.randn((2, 4, 64, 16), generator=g)
    assert torch.equal(q, q32.to(torch.bfloat16))


def test_heavy_keys_scale_one_percent_of_rows():
    w = synthetic.custom("t", "fp32", 1, 2, 1, 1000, 8, 4, True, "striped", 3, heavy_keys=True)
    _, k, _ = synthetic.make_inputs(w, "cpu")
    g = torch.Generator().manual_seed(3)
    torch.randn((1, 2, 1000, 8), generator=g)
    k0 = torch.randn((1, 1, 1000, 8), generator=g)
    torch.randn((1, 1, 1000, 8), generator=g)
    idx = torch.randperm(1000, generator=g)[: int(math.floor(0.01 * 1000))]
    ratio = (k[0, 0] / k0[0, 0])
    heavy = torch.zeros(1000, dtype=torch.bool)
    heavy[idx] = True
    assert torch.allclose(ratio[heavy], torch.full_like(ratio[heavy], 4.0))
    assert torch.allclose(ratio[~heavy], torch.ones_like(ratio[~heavy]))


def test_sampled_rows_include_boundaries_and_are_seeded():
    w = synthetic.get("c5_bf16_s1m_striped")
    r1 = synthetic.sample_rows(w, 256)
    r2 = synthetic.sample_rows(w, 256)
    assert r1 == r2
    for row in synthetic.shard_boundary_rows(w):
        assert row in r1
    assert (0, 0, 0) in r1 and (0, 0, w.S - 1) in r1
    assert all(0 <= b < w.B and 0 <= h < w.Hq and 0 <= t < w.S for b, h, t in r1)


def test_workload_table_matches_flop_formula():
    w = synthetic.get("c5_bf16_s1m_striped")
    assert w.causal_flops() == 2.0 ** 51
    assert synthetic.get("c4_bf16_gqa_s128k").causal_flops() == 2.0 ** 48
    for w in synthetic.WORKLOADS.values():
        assert w.S % w.P == 0 and w.Hq % w.Hkv == 0
