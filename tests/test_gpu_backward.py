"""GPU: the backward pass (ring_attn_bwd through the C ABI) against the fp64 backward oracle.

Tolerance. The gradients are bf16 and the kernels round P and dS to bf16 before
their tensor-core products (as the forward rounds P), so each term carries about
2^-9 relative error on top of the bf16 rounding of the result. The check is per
gradient tensor: max |got - ref| <= 2e-2 * max |ref| and rms(got - ref) <= 1e-2 * rms(ref).
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from sequence_exact_attention_ring_b200 import binding, ring_attention, ring_attention_backward

pytestmark = pytest.mark.gpu

MAX_REL, RMS_REL = 2e-2, 1e-2


def assert_grad(got, ref, what):
    g = got.float().cpu().numpy().astype(np.float64) if isinstance(got, torch.Tensor) else got
    d = g - ref
    scale = np.abs(ref).max()
    assert np.isfinite(g).all(), f"{what}: non-finite"
    assert np.abs(d).max() <= MAX_REL * scale, f"{what}: max|d|={np.abs(d).max():.3e} max|ref|={scale:.3e}"
    rms = np.sqrt(np.mean(d * d))
    assert rms <= RMS_REL * np.sqrt(np.mean(ref * ref)), f"{what}: rms(d)={rms:.3e}"


def make(B, Hq, Hkv, S, D, P, causal, layout, seed, device="cpu"):
    w = synthetic.custom("bwd", "bf16", B, Hq, Hkv, S, D, P, causal, layout, seed, gen_device=device)
    q, k, v = (t.cuda() for t in synthetic.make_inputs(w, device))
    dout = synthetic.make_dout(w, device).cuda()
    out, lse = ring_attention(q, k, v, P, causal, layout, w.scale)
    return w, q, k, v, dout, out, lse


CASES = [
    # (B, Hq, Hkv, S, D, P, causal, layout): several tiles, ragged tails, GQA, every layout
    (1, 2, 2, 512, 128, 4, True, "striped"),
    (1, 2, 2, 640, 128, 4, True, "contiguous"),   # Sq = 160: ragged query and key tiles
    (2, 4, 2, 768, 128, 3, True, "striped"),      # GQA 2, B = 2, Sq = 256
    (1, 2, 2, 1024, 128, 4, False, "contiguous"),
    (1, 2, 2, 1024, 128, 4, True, "zigzag"),      # C = 128
    (1, 2, 2, 384, 128, 1, True, "contiguous"),   # P = 1: plain causal attention
    (1, 8, 1, 512, 128, 8, True, "striped"),      # GQA 8: dK, dV sum over 8 query heads
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_backward_small_cases_all_elements(cuda_lib, case):
    w, q, k, v, dout, out, lse = make(*case, seed=201)
    dq, dk, dv = ring_attention_backward(q, k, v, out, lse, dout, w.P, w.causal, w.layout, w.scale)
    torch.cuda.synchronize()
    ref = oracle.attention_backward_reference(q.cpu(), k.cpu(), v.cpu(), dout.cpu(), w.causal, w.scale)
    for name, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        assert_grad(got, r, f"{case} {name}")


def test_backward_layouts_agree(cuda_lib):
    """Layout only changes the schedule: the three layouts give the same gradients."""
    res = {}
    for layout in ("contiguous", "striped", "zigzag"):
        w, q, k, v, dout, out, lse = make(1, 4, 2, 2048, 128, 8, True, layout, seed=211)
        res[layout] = [t.float() for t in ring_attention_backward(q, k, v, out, lse, dout, w.P, True, layout)]
    for layout in ("striped", "zigzag"):
        for a, b in zip(res[layout], res["contiguous"]):
            assert (a - b).abs().max().item() <= MAX_REL * b.abs().max().item(), layout


@pytest.mark.parametrize("name", ["c3_bf16_s16k_striped", "c2_bf16_s16k_contig"])
def test_backward_16k_sampled(cuda_lib, name):
    """16k tokens: sampled dQ rows, the last keys' dK/dV exactly, column sums for all keys."""
    w0 = synthetic.get(name)
    w, q, k, v, dout, out, lse = make(w0.B, w0.Hq, w0.Hkv, w0.S, w0.D, w0.P, w0.causal, w0.layout, w0.seed)
    dq, dk, dv = ring_attention_backward(q, k, v, out, lse, dout, w.P, w.causal, w.layout, w.scale)
    torch.cuda.synchronize()
    qh, kh, vh, doh = q.cpu(), k.cpu(), v.cpu(), dout.cpu()
    rows = synthetic.sample_rows(w, 256)
    ref_q = oracle.backward_rows_dq(qh, kh, vh, doh, rows, w.causal, w.scale)
    got_q = torch.stack([dq[b, h, t] for b, h, t in rows])
    assert_grad(got_q, ref_q, f"{name} dq rows")
    keys = [(0, g, u) for g in range(w.Hkv) for u in range(w.S - 48, w.S)]
    ref_k, ref_v = oracle.backward_rows_dkdv(qh, kh, vh, doh, keys, w.causal, w.scale)
    got_k = torch.stack([dk[b, g, u] for b, g, u in keys])
    got_v = torch.stack([dv[b, g, u] for b, g, u in keys])
    assert_grad(got_k, ref_k, f"{name} dk late keys")
    assert_grad(got_v, ref_v, f"{name} dv late keys")
    # every row of P sums to 1 and every row of dS to 0: sum_u dV_u = sum_t dO_t, sum_u dK_u = 0
    sv = dv.double().sum(dim=2).cpu().numpy()
    so = dout.double().sum(dim=2).cpu().numpy()
    assert np.abs(sv - so).max() <= 2e-2 * dv.double().abs().sum(dim=2).max().item()
    sk = dk.double().sum(dim=2).cpu().numpy()
    assert np.abs(sk).max() <= 2e-2 * dk.double().abs().sum(dim=2).max().item()


# shapes the tensor-core kernels do not take run on the CUDA-core backward
SIMT_CASES = [
    # (B, Hq, Hkv, S, D, P, causal, layout, dtype)
    (1, 2, 2, 1000, 128, 4, True, "zigzag", "bf16"),     # C = 125: not whole 128-row tiles
    (1, 4, 2, 768, 64, 3, True, "striped", "bf16"),      # D = 64
    (1, 2, 1, 640, 64, 4, True, "contiguous", "fp32"),   # fp32, ragged Sq = 160
    (2, 2, 2, 512, 128, 2, False, "striped", "fp32"),
]


@pytest.mark.parametrize("case", SIMT_CASES, ids=lambda c: "-".join(map(str, c)))
def test_backward_cuda_core_path(cuda_lib, case):
    B, Hq, Hkv, S, D, P, causal, layout, dtype = case
    w = synthetic.custom("bwd", dtype, B, Hq, Hkv, S, D, P, causal, layout, 231)
    q, k, v = (t.cuda() for t in synthetic.make_inputs(w, "cpu"))
    dout = synthetic.make_dout(w, "cpu").cuda()
    out, lse = ring_attention(q, k, v, P, causal, layout, w.scale)
    dq, dk, dv = ring_attention_backward(q, k, v, out, lse, dout, P, causal, layout, w.scale)
    torch.cuda.synchronize()
    ref = oracle.attention_backward_reference(q.cpu(), k.cpu(), v.cpu(), dout.cpu(), causal, w.scale)
    for name, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        if dtype == "fp32":
            # fp32 throughout (exact exp2f, no rounded P): relative to the largest gradient
            g = got.cpu().numpy().astype(np.float64)
            assert np.abs(g - r).max() <= 1e-4 * np.abs(r).max(), f"{case} {name}"
        else:
            assert_grad(got, r, f"{case} {name}")


# ------------------------------------------------------------------ long sequences
# From S*D >= 2^23 (S >= 65536 at D = 128) the dK/dV and dQ kernels switch to their
# grouped launch orders, the regime the backward benchmark runs. Every element of
# dq, dk and dv is compared with the fp64 oracle at 64k tokens, for the three layouts.

LONG_CASES = [
    # (B, Hq, Hkv, S, D, P, causal, layout)
    (1, 1, 1, 65536, 128, 8, True, "contiguous"),
    (1, 1, 1, 65536, 128, 8, True, "striped"),
    (1, 1, 1, 65536, 128, 8, True, "zigzag"),   # C = 4096: whole 128-row tiles
]


@pytest.mark.parametrize("case", LONG_CASES, ids=lambda c: f"{c[7]}-S{c[3]}")
def test_backward_64k_all_elements(cuda_lib, case):
    w, q, k, v, dout, out, lse = make(*case, seed=241)
    dq, dk, dv = ring_attention_backward(q, k, v, out, lse, dout, w.P, w.causal, w.layout, w.scale)
    torch.cuda.synchronize()
    ref = oracle.attention_backward_reference(q.cpu(), k.cpu(), v.cpu(), dout.cpu(), w.causal, w.scale)
    for name, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        assert_grad(got, r, f"{case} {name}")


def test_backward_c4_gqa_heavy_keys_sampled(cuda_lib):
    """The 131k GQA workload with heavy keys (striped, P = 16, 4 query heads per kv head):
    1024 seeded dQ rows plus the shard-boundary rows; dK/dV of the last 64 tokens of
    every (batch, kv head), which hold the last key of every shard; column sums over all keys."""
    w = synthetic.get("c4_bf16_gqa_s128k")
    q, k, v = synthetic.make_inputs(w, "cuda")
    dout = synthetic.make_dout(w, "cuda")
    out, lse = ring_attention(q, k, v, w.P, w.causal, w.layout, w.scale)
    dq, dk, dv = ring_attention_backward(q, k, v, out, lse, dout, w.P, w.causal, w.layout, w.scale)
    torch.cuda.synchronize()
    qh, kh, vh, doh = q.cpu(), k.cpu(), v.cpu(), dout.cpu()
    rows = synthetic.sample_rows(w, 1024)
    ref_q = oracle.backward_rows_dq(qh, kh, vh, doh, rows, w.causal, w.scale)
    got_q = torch.stack([dq[b, h, t] for b, h, t in rows])
    assert_grad(got_q, ref_q, "c4 dq rows")
    keys = [(b, g, u) for b in range(w.B) for g in range(w.Hkv) for u in range(w.S - 64, w.S)]
    ref_k, ref_v = oracle.backward_rows_dkdv(qh, kh, vh, doh, keys, w.causal, w.scale)
    got_k = torch.stack([dk[b, g, u] for b, g, u in keys])
    got_v = torch.stack([dv[b, g, u] for b, g, u in keys])
    assert_grad(got_k, ref_k, "c4 dk last keys")
    assert_grad(got_v, ref_v, "c4 dv last keys")
    # every row of P sums to 1 and every row of dS to 0, per kv head over its query heads:
    # sum_u dV_u = sum over the group's rows of dO_t, and sum_u dK_u = 0
    rep = w.Hq // w.Hkv
    sv = dv.double().sum(dim=2)
    so = dout.double().view(w.B, w.Hkv, rep, w.S, w.D).sum(dim=(2, 3))
    assert (sv - so).abs().max().item() <= 2e-2 * dv.double().abs().sum(dim=2).max().item()
    sk = dk.double().sum(dim=2)
    assert sk.abs().max().item() <= 2e-2 * dk.double().abs().sum(dim=2).max().item()
