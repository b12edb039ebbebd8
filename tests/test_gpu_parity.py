"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Every comparison uses identical seeded inputs (the oracle reads exact fp64
copies of the rounded device tensors) and the tolerances of the workload spec.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic
from gpu_helpers import assert_parity, gather_rows
from sequence_exact_attention_ring_b200 import ring_attention

pytestmark = pytest.mark.gpu

SMALL = [
    # (B, Hq, Hkv, S, D, P, causal, layout, dtype, algo)  several tiles + ragged tails
    (1, 2, 2, 1024, 64, 4, False, "contiguous", "fp32", "auto"),
    (1, 2, 1, 800, 128, 4, True, "striped", "fp32", "auto"),        # Sq=200: ragged q and kv tiles
    (1, 2, 2, 800, 128, 4, True, "contiguous", "bf16", "tcgen05"),
    (1, 2, 2, 800, 128, 4, True, "striped", "bf16", "tcgen05"),
    (2, 4, 2, 1536, 128, 3, True, "striped", "bf16", "tcgen05"),     # Sq=512, GQA 2, B=2
    (1, 8, 1, 1024, 128, 8, True, "contiguous", "bf16", "tcgen05"),  # GQA 8
    (1, 4, 4, 1280, 64, 5, True, "striped", "bf16", "tcgen05"),      # D=64
    (1, 2, 2, 2048, 128, 1, True, "contiguous", "bf16", "tcgen05"),  # P=1: plain causal attention
    (1, 2, 2, 96, 128, 96, True, "striped", "bf16", "tcgen05"),      # P=S: one token per shard
    (1, 2, 2, 1000, 128, 8, False, "striped", "bf16", "tcgen05"),    # non-causal, Sq=125
    (1, 2, 2, 800, 128, 4, True, "striped", "bf16", "tcgen05_1sm"),
    (2, 4, 2, 1536, 128, 3, True, "contiguous", "bf16", "tcgen05_1sm"),
    (1, 2, 2, 1000, 128, 8, False, "striped", "bf16", "tcgen05_1sm"),
    (1, 2, 2, 1100, 128, 1, True, "contiguous", "bf16", "tcgen05"),    # ragged tail inside a 512-row pair block
    (1, 3, 3, 640, 128, 2, True, "striped", "bf16", "simt"),
    (1, 2, 2, 384, 64, 4, False, "contiguous", "bf16", "simt"),
    # zigzag: shard i = chunks i and 2P-1-i of C = S/(2P) tokens
    (1, 2, 2, 2048, 128, 4, True, "zigzag", "bf16", "tcgen05"),      # C=256: 512-row units span two chunks
    (2, 4, 2, 3072, 128, 3, True, "zigzag", "bf16", "tcgen05"),      # C=512: chunk-ordered units, GQA 2
    (1, 2, 2, 1024, 128, 4, False, "zigzag", "bf16", "tcgen05"),     # C=128, non-causal
    (1, 4, 4, 2560, 64, 5, True, "zigzag", "bf16", "tcgen05"),       # D=64
    (1, 2, 2, 2048, 128, 4, True, "zigzag", "bf16", "tcgen05_1sm"),
    (1, 2, 2, 1000, 128, 4, True, "zigzag", "bf16", "auto"),         # C=125: AUTO takes the SIMT kernel
    (1, 2, 2, 640, 64, 4, True, "zigzag", "fp32", "auto"),
]


def run_case(B, Hq, Hkv, S, D, P, causal, layout, dtype, algo, seed=123):
    w = synthetic.custom("case", dtype, B, Hq, Hkv, S, D, P, causal, layout, seed)
    q, k, v = (t.cuda() for t in synthetic.make_inputs(w, "cpu"))
    out, lse = ring_attention(q, k, v, P, causal, layout, w.scale, algo=algo)
    torch.cuda.synchronize()
    return w, q, k, v, out, lse


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "-".join(map(str, c)))
def test_small_cases_all_rows(cuda_lib, case):
    w, q, k, v, out, lse = run_case(*case)
    O_ref, L_ref = oracle.attention_reference(q.cpu(), k.cpu(), v.cpu(), w.causal, w.scale)
    assert_parity(out, lse, O_ref, L_ref, w.torch_dtype, str(case))


def test_c1_fp32_all_rows(cuda_lib):
    w = synthetic.get("c1_fp32_s1k")
    q, k, v = (t.cuda() for t in synthetic.make_inputs(w))
    out, lse = ring_attention(q, k, v, w.P, w.causal, w.layout, w.scale)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle.attention_reference(q.cpu(), k.cpu(), v.cpu(), w.causal, w.scale)
    assert_parity(out, lse, O_ref, L_ref, torch.float32, w.name)


@pytest.mark.parametrize("name", ["c2_bf16_s16k_contig", "c3_bf16_s16k_striped"])
def test_16k_configs_all_rows(cuda_lib, name):
    w = synthetic.get(name)
    q, k, v = (t.cuda() for t in synthetic.make_inputs(w))
    out, lse = ring_attention(q, k, v, w.P, w.causal, w.layout, w.scale)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle.attention_reference(q.cpu(), k.cpu(), v.cpu(), w.causal, w.scale)
    assert_parity(out, lse, O_ref, L_ref, torch.bfloat16, name)


def test_layouts_and_kernels_agree(cuda_lib):
    """Layout and kernel choice only change the schedule: outputs agree with each other."""
    base = (1, 4, 2, 2048, 128, 8, True)
    res = {}
    for layout in ("contiguous", "striped", "zigzag"):
        for algo in ("tcgen05", "tcgen05_1sm", "simt"):
            _, _, _, _, out, lse = run_case(*base, layout, "bf16", algo, seed=77)
            res[(layout, algo)] = (out.float(), lse)
    ref_o, ref_l = res[("contiguous", "simt")]
    for key, (o, l) in res.items():
        assert (o - ref_o).abs().max().item() <= 2e-2, key
        assert ((l - ref_l).abs() / ref_l.abs().clamp_min(1)).max().item() <= 1e-3, key


def test_zigzag_chunks_the_tensor_cores_cannot_tile_are_refused(cuda_lib):
    from sequence_exact_attention_ring_b200 import binding
    w = synthetic.custom("zz", "bf16", 1, 2, 2, 1000, 128, 4, True, "zigzag", 1)
    q, k, v = (t.cuda() for t in synthetic.make_inputs(w, "cpu"))
    with pytest.raises(binding.RingAttnError) as e:
        ring_attention(q, k, v, w.P, True, "zigzag", w.scale, algo="tcgen05")
    assert e.value.code == binding.EUNSUPPORTED


@pytest.mark.parametrize("name", ["c4_bf16_gqa_s128k", "c5_bf16_s1m_striped", "z5_bf16_s1m_zigzag"])
def test_large_configs_sampled_rows(cuda_lib, name):
    """Full-size launch (as the benchmark runs it), checked on 4096 seeded rows + shard boundaries."""
    w = synthetic.get(name)
    q, k, v = synthetic.make_inputs(w, "cuda")
    out, lse = ring_attention(q, k, v, w.P, w.causal, w.layout, w.scale)
    torch.cuda.synchronize()
    rows = synthetic.sample_rows(w, 4096)
    o_s, l_s = gather_rows(out, lse, rows)
    qh, kh, vh = q.cpu(), k.cpu(), v.cpu()
    O_ref, L_ref = oracle.attention_rows(qh, kh, vh, rows, w.causal, w.scale)
    assert_parity(o_s, l_s, O_ref, L_ref, torch.bfloat16, name)


@pytest.mark.parametrize("D,algo", [(128, "tcgen05"), (64, "tcgen05"), (128, "tcgen05_1sm")])
@pytest.mark.parametrize("pattern", ["rising", "jump"])
def test_reference_maximum_moves(cuda_lib, D, algo, pattern):
    """Scores that climb along the sequence (the running maximum moves again and again), or
    a few keys whose scores jump far past 2^127 relative to the running maximum (one block's
    exponentials overflow): the kernels exponentiate against the running maximum first and
    must fall back to the block maximum and rescale O and l."""
    w = synthetic.custom("mx", "bf16", 1, 2, 2, 2048, D, 4, True, "striped", 41)
    q, k, v = synthetic.make_inputs(w, "cpu")
    kf = k.float()
    if pattern == "rising":
        kf = kf * (1.0 + 6.0 * torch.arange(w.S, dtype=torch.float32) / w.S)[None, None, :, None]
    else:
        idx = torch.randperm(w.S, generator=torch.Generator().manual_seed(5))[:8]
        kf[:, :, idx] *= 128.0
    k = kf.to(torch.bfloat16)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    out, lse = ring_attention(q, k, v, w.P, True, "striped", w.scale, algo=algo)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle.attention_reference(q.cpu(), k.cpu(), v.cpu(), True, w.scale)
    assert_parity(out, lse, O_ref, L_ref, torch.bfloat16, f"{pattern} D={D} {algo}")
