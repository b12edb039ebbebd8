"""GPU: decode against a sharded KV cache (ring_attn_decode through the C ABI) vs the fp64 oracle.

Tolerances are the forward's bf16 ones (max |dO| <= 2e-2, lse relative <= 1e-3).
"""
import pytest
import torch

import oracle
import synthetic
from gpu_helpers import assert_parity
from sequence_exact_attention_ring_b200 import binding, ring_attention_decode

pytestmark = pytest.mark.gpu

CASES = [
    # (B, Hq, Hkv, S, P, layout)
    (1, 2, 2, 1024, 4, "striped"),
    (2, 8, 2, 3000, 3, "contiguous"),   # Sq = 1000: ragged last tile of every shard
    (1, 16, 1, 2048, 8, "zigzag"),      # C = 128; 16 query heads share one kv head
    (2, 64, 2, 1536, 3, "striped"),     # 32 query heads per kv head (the largest group)
    (1, 4, 1, 640, 5, "contiguous"),    # Sq = 128: one tile per shard
    (1, 4, 4, 512, 1, "contiguous"),    # P = 1
    (1, 8, 8, 65536, 32, "striped"),
]


def run(B, Hq, Hkv, S, P, layout, seed, device="cpu", heavy=False):
    w = synthetic.custom("dec", "bf16", B, Hq, Hkv, S, 128, P, False, layout, seed, heavy, device)
    _, k, v = synthetic.make_inputs(w, device)
    q1 = synthetic.make_decode_query(w, device)
    k, v, q1 = k.cuda(), v.cuda(), q1.cuda()
    out, lse = ring_attention_decode(q1, k, v, P, layout, w.scale)
    torch.cuda.synchronize()
    return w, q1, k, v, out, lse


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_decode_against_oracle(cuda_lib, case):
    w, q1, k, v, out, lse = run(*case, seed=301)
    O_ref, L_ref = oracle.decode_reference(q1.cpu(), k.cpu(), v.cpu(), w.scale)
    assert_parity(out, lse, O_ref, L_ref, torch.bfloat16, str(case))


def test_decode_1m_cache_with_heavy_keys(cuda_lib):
    """The 1M-token cache of the benchmark workload's shape, 1% of keys scaled by 4."""
    w, q1, k, v, out, lse = run(1, 8, 8, 1 << 20, 32, "striped", seed=311, device="cuda", heavy=True)
    O_ref, L_ref = oracle.decode_reference(q1.cpu(), k.cpu(), v.cpu(), w.scale)
    assert_parity(out, lse, O_ref, L_ref, torch.bfloat16, "1M cache")


def test_decode_layouts_agree_and_refusals(cuda_lib):
    res = [run(1, 4, 2, 4096, 4, layout, seed=321)[4:] for layout in ("contiguous", "striped", "zigzag")]
    for o, l in res[1:]:
        assert (o.float() - res[0][0].float()).abs().max().item() <= 2e-2
        assert ((l - res[0][1]).abs() / res[0][1].abs().clamp_min(1)).max().item() <= 1e-3
    w = synthetic.custom("dec", "bf16", 1, 2, 2, 1000, 128, 4, False, "zigzag", 1)
    _, k, v = (t.cuda() for t in synthetic.make_inputs(w, "cpu"))
    with pytest.raises(binding.RingAttnError) as e:
        ring_attention_decode(synthetic.make_decode_query(w, "cpu").cuda(), k, v, 4, "zigzag")
    assert e.value.code == binding.EUNSUPPORTED
