"""GPU: the ring step on shard-local buffers (ring_attn_fwd_ring_step through the C ABI),
the whole ring run step by step, and the virtual ring (P ranks on one device with their
own buffers, streams and device-to-device transfers), all against the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gpu_helpers import assert_parity
from sequence_exact_attention_ring_b200 import RingAttnError, binding, ring, ring_attention_ring_step

pytestmark = pytest.mark.gpu


def shards_of(w, q, k, v):
    return (ring.split_shards(q, w.P, w.layout), ring.split_shards(k, w.P, w.layout),
            ring.split_shards(v, w.P, w.layout))


def run_ring_sequential(w, qs, ks, vs):
    """Every rank's P steps, one after another on one stream, in the ring order of
    section 2: rank r holds KV shard (r - s) mod P at step s."""
    outs, lses = [], []
    for r in range(w.P):
        B, Hq, Sq, D = qs[r].shape
        o_acc = torch.full((B, Hq, Sq, D), float("nan"), dtype=torch.float32, device="cuda")
        l_acc = torch.full((B, Hq, Sq), float("nan"), dtype=torch.float32, device="cuda")
        out = lse = None
        for s in range(w.P):
            j = (r - s) % w.P
            res = ring_attention_ring_step(qs[r], ks[j], vs[j], w.S, w.P, r, j, w.causal, w.layout, w.scale,
                                           first=s == 0, last=s == w.P - 1, o_acc=o_acc, lse_acc=l_acc)
            if s == w.P - 1:
                out, lse = res
        outs.append(out)
        lses.append(lse)
    return ring.join_shards(outs, w.layout), ring.join_shards(lses, w.layout)


CASES = [
    # (dtype, B, Hq, Hkv, S, D, P, causal, layout)
    ("bf16", 1, 4, 2, 2048, 128, 4, True, "striped"),
    ("bf16", 1, 4, 2, 2048, 128, 4, True, "contiguous"),    # steps j > i are fully masked
    ("bf16", 1, 2, 2, 2048, 128, 4, True, "zigzag"),
    ("bf16", 2, 4, 4, 1536, 128, 3, False, "striped"),
    ("bf16", 1, 2, 1, 1000, 128, 4, True, "zigzag"),        # C = 125: not whole tiles, runs on the tensor cores here
    ("bf16", 1, 2, 2, 1280, 64, 5, True, "striped"),        # D = 64: the single-CTA kernel
    ("fp32", 1, 2, 2, 1024, 64, 4, False, "contiguous"),    # the CUDA-core kernel
    ("fp32", 1, 2, 1, 768, 128, 3, True, "striped"),
    ("bf16", 1, 2, 2, 1024, 128, 1, True, "striped"),       # P = 1: first and last in one step
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_ring_steps_fold_to_the_oracle(cuda_lib, case):
    dtype, B, Hq, Hkv, S, D, P, causal, layout = case
    w = synthetic.custom("ring", dtype, B, Hq, Hkv, S, D, P, causal, layout, 301)
    q, k, v = (t.cuda() for t in synthetic.make_inputs(w, "cpu"))
    out, lse = run_ring_sequential(w, *shards_of(w, q, k, v))
    torch.cuda.synchronize()
    O_ref, L_ref = oracle.attention_reference(q.cpu(), k.cpu(), v.cpu(), causal, w.scale)
    assert_parity(out, lse, O_ref, L_ref, q.dtype, str(case))


def test_virtual_ring_matches_the_oracle(cuda_lib):
    """P = 4 virtual ranks on one device: transfers on copy streams, steps on compute streams."""
    for layout in ("striped", "contiguous"):
        w = synthetic.custom("vring", "bf16", 1, 4, 2, 4096, 128, 4, True, layout, 311)
        q, k, v = (t.cuda() for t in synthetic.make_inputs(w, "cpu"))
        vr = ring.VirtualRing(*shards_of(w, q, k, v), causal=True, layout=layout, scale=w.scale)
        vr.run()
        torch.cuda.synchronize()
        res = vr.results()
        out = ring.join_shards([o for o, _ in res], layout)
        lse = ring.join_shards([l for _, l in res], layout)
        O_ref, L_ref = oracle.attention_reference(q.cpu(), k.cpu(), v.cpu(), True, w.scale)
        assert_parity(out, lse, O_ref, L_ref, torch.bfloat16, f"virtual ring {layout}")
        for ws in vr.ws:
            assert binding.ring_attn_status(ws.data_ptr(), torch.cuda.current_stream().cuda_stream) == 0
        # the caller's shards are untouched by the transfers
        for r, (kr, vr_) in enumerate(zip(*shards_of(w, q, k, v)[1:])):
            assert torch.equal(vr.k[r], kr) and torch.equal(vr.v[r], vr_)


def test_virtual_ring_twice_in_a_row_is_identical(cuda_lib):
    """A second run reuses every buffer; the result is bit-identical."""
    w = synthetic.custom("vring2", "bf16", 1, 2, 2, 2048, 128, 8, True, "striped", 313)
    q, k, v = (t.cuda() for t in synthetic.make_inputs(w, "cpu"))
    vr = ring.VirtualRing(*shards_of(w, q, k, v), causal=True, layout="striped", scale=w.scale)
    vr.run()
    first = [(o.clone(), l.clone()) for o, l in vr.results()]
    vr.run(timing=True)
    torch.cuda.synchronize()
    for (o1, l1), (o2, l2) in zip(first, vr.results()):
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_ring_step_matches_the_partial_step_and_merge(cuda_lib):
    """Folding the P steps of one query shard equals merging the P normalised partials
    of ring_attn_fwd_step with ring_attn_merge (two routes to the section 3 rescale)."""
    from sequence_exact_attention_ring_b200 import merge, ring_attention_step
    w = synthetic.custom("fold", "bf16", 1, 4, 2, 2048, 128, 4, True, "striped", 317)
    q, k, v = (t.cuda() for t in synthetic.make_inputs(w, "cpu"))
    qs, ks, vs = shards_of(w, q, k, v)
    i = 2
    parts = [ring_attention_step(q, k, v, w.P, i, j, True, "striped", w.scale) for j in range(w.P)]
    o_m, l_m = merge(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]), torch.float32)
    o_acc = torch.empty_like(o_m)
    l_acc = torch.empty_like(l_m)
    for s in range(w.P - 1):
        j = (i - s) % w.P
        ring_attention_ring_step(qs[i], ks[j], vs[j], w.S, w.P, i, j, True, "striped", w.scale, first=s == 0,
                                 o_acc=o_acc, lse_acc=l_acc)
    torch.cuda.synchronize()
    # after P - 1 steps the state is the merge of those P - 1 partials
    o_m3, l_m3 = merge(torch.stack([parts[(i - s) % w.P][0] for s in range(w.P - 1)]),
                       torch.stack([parts[(i - s) % w.P][1] for s in range(w.P - 1)]), torch.float32)
    assert (o_acc - o_m3).abs().max().item() <= 1e-5
    assert (l_acc - l_m3).abs().max().item() <= 1e-5
    j = (i - (w.P - 1)) % w.P
    out, lse = ring_attention_ring_step(qs[i], ks[j], vs[j], w.S, w.P, i, j, True, "striped", w.scale, last=True,
                                        o_acc=o_acc, lse_acc=l_acc)
    torch.cuda.synchronize()
    assert (out.float() - o_m).abs().max().item() <= 2e-2
    assert (lse - l_m).abs().max().item() <= 1e-5
    assert np.isfinite(lse.cpu().numpy()).all()


def test_ring_step_rejects_bad_arguments(cuda_lib):
    w = synthetic.custom("bad", "bf16", 1, 2, 2, 1024, 128, 4, True, "striped", 319)
    q, k, v = (t.cuda() for t in synthetic.make_inputs(w, "cpu"))
    qs, ks, vs = shards_of(w, q, k, v)
    with pytest.raises(ValueError):     # a step that is not both first and last needs the state
        ring_attention_ring_step(qs[0], ks[0], vs[0], w.S, w.P, 0, 0, True, "striped", w.scale)
    with pytest.raises(ValueError):     # shard length must be S / P
        ring_attention_ring_step(qs[0], ks[0], vs[0], w.S + 4, w.P, 0, 0, True, "striped", w.scale, first=True,
                                 last=True)
    with pytest.raises(RingAttnError):  # kv_index out of range
        ring_attention_ring_step(qs[0], ks[0], vs[0], w.S, w.P, 0, 4, True, "striped", w.scale, first=True,
                                 last=True)


# ------------------------------------------------------------------ backward ring

def run_backward_ring_sequential(w, q, k, v, out, lse, dout):
    """Every rank's steps of the backward ring, one after another on one stream: rank r
    (query shard r) holds KV shard (r + s) mod P at step s; the dK/dV accumulators belong
    to the KV shard and are handed from rank to rank, the dQ accumulator stays at its rank."""
    from sequence_exact_attention_ring_b200 import ring_backward_prep, ring_backward_step
    P = w.P
    qs, ks, vs, douts = (ring.split_shards(t, P, w.layout) for t in (q, k, v, dout))
    outs = ring.split_shards(out, P, w.layout)
    lses = [x.contiguous() for x in ring.split_shards(lse.unsqueeze(-1), P, w.layout)]
    lses = [x.squeeze(-1).contiguous() for x in lses]
    wss = [ring_backward_prep(outs[r], lses[r], douts[r], w.S, P, r, w.causal, w.layout) for r in range(P)]
    f32 = dict(dtype=torch.float32, device="cuda")
    dq_acc = [torch.full(x.shape, float("nan"), **f32) for x in qs]
    dk_acc = [torch.full(x.shape, float("nan"), **f32) for x in ks]
    dv_acc = [torch.full(x.shape, float("nan"), **f32) for x in vs]
    dq = [torch.empty_like(x) for x in qs]
    dk = [torch.empty_like(x) for x in ks]
    dv = [torch.empty_like(x) for x in vs]
    for s in range(P):
        for r in range(P):
            j = (r + s) % P
            ring_backward_step(qs[r], douts[r], ks[j], vs[j], w.S, P, r, j, wss[r], w.causal, w.layout, w.scale,
                               parts=3, first=s == 0, last=s == P - 1, dq_acc=dq_acc[r], dk_acc=dk_acc[j],
                               dv_acc=dv_acc[j], dq=dq[r], dk=dk[j], dv=dv[j])
    return (ring.join_shards(dq, w.layout), ring.join_shards(dk, w.layout), ring.join_shards(dv, w.layout))


BWD_RING_CASES = [
    # (B, Hq, Hkv, S, P, causal, layout)
    (1, 2, 2, 1024, 4, True, "striped"),
    (1, 2, 2, 1024, 4, True, "contiguous"),    # steps with j > i see nothing
    (2, 4, 2, 768, 3, True, "striped"),        # GQA 2, B = 2
    (1, 2, 2, 1024, 4, True, "zigzag"),
    (1, 2, 1, 1000, 4, True, "zigzag"),        # C = 125: not whole tiles
    (1, 2, 2, 1024, 4, False, "contiguous"),
    (1, 2, 2, 640, 1, True, "striped"),        # P = 1: first and last in one step
]


@pytest.mark.parametrize("case", BWD_RING_CASES, ids=lambda c: "-".join(map(str, c)))
def test_backward_ring_steps_match_the_oracle(cuda_lib, case):
    from test_gpu_backward import assert_grad
    from sequence_exact_attention_ring_b200 import ring_attention
    B, Hq, Hkv, S, P, causal, layout = case
    w = synthetic.custom("bring", "bf16", B, Hq, Hkv, S, 128, P, causal, layout, 331)
    q, k, v = (t.cuda() for t in synthetic.make_inputs(w, "cpu"))
    dout = synthetic.make_dout(w, "cpu").cuda()
    out, lse = ring_attention(q, k, v, P, causal, layout, w.scale)
    dq, dk, dv = run_backward_ring_sequential(w, q, k, v, out, lse, dout)
    torch.cuda.synchronize()
    ref = oracle.attention_backward_reference(q.cpu(), k.cpu(), v.cpu(), dout.cpu(), causal, w.scale)
    for name, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        assert_grad(got, r, f"{case} {name}")


def test_backward_ring_parts_called_separately_agree(cuda_lib):
    """Running the dK/dV part and the dQ part as two calls (so the accumulators can leave
    between them) gives the same bits as one call with both parts."""
    from sequence_exact_attention_ring_b200 import ring_attention, ring_backward_prep, ring_backward_step
    w = synthetic.custom("bparts", "bf16", 1, 2, 2, 1024, 128, 4, True, "striped", 337)
    q, k, v = (t.cuda() for t in synthetic.make_inputs(w, "cpu"))
    dout = synthetic.make_dout(w, "cpu").cuda()
    out, lse = ring_attention(q, k, v, w.P, True, "striped", w.scale)
    qs, ks, vs, douts, outs = (ring.split_shards(t, w.P, "striped") for t in (q, k, v, dout, out))
    lses = [x.squeeze(-1).contiguous() for x in ring.split_shards(lse.unsqueeze(-1), w.P, "striped")]
    r, j = 1, 3
    ws = ring_backward_prep(outs[r], lses[r], douts[r], w.S, w.P, r, True, "striped")
    res = []
    for split in (False, True):
        accs = [torch.zeros(x.shape, dtype=torch.float32, device="cuda") for x in (qs[r], ks[j], vs[j])]
        kw = dict(first=True, dq_acc=accs[0], dk_acc=accs[1], dv_acc=accs[2])
        if split:
            ring_backward_step(qs[r], douts[r], ks[j], vs[j], w.S, w.P, r, j, ws, True, "striped", w.scale, parts=1, **kw)
            ring_backward_step(qs[r], douts[r], ks[j], vs[j], w.S, w.P, r, j, ws, True, "striped", w.scale, parts=2, **kw)
        else:
            ring_backward_step(qs[r], douts[r], ks[j], vs[j], w.S, w.P, r, j, ws, True, "striped", w.scale, parts=3, **kw)
        torch.cuda.synchronize()
        res.append([a.clone() for a in accs])
        assert all(torch.isfinite(a).all() for a in accs)
    for a, b in zip(*res):
        assert torch.equal(a, b)


@pytest.mark.parametrize("layout,P", [("striped", 4), ("contiguous", 4), ("striped", 1)])
def test_virtual_backward_ring_matches_the_oracle(cuda_lib, layout, P):
    """P virtual ranks of the backward ring on one device: K/V and the dK/dV accumulators
    travel by device-to-device copies on copy streams while the step kernels run; the
    gradients against the fp64 oracle, and a second (timed) run bit-identical."""
    from test_gpu_backward import assert_grad
    from sequence_exact_attention_ring_b200 import ring_attention
    w = synthetic.custom("vbring", "bf16", 1, 4, 2, 2048, 128, P, True, layout, 341)
    q, k, v = (t.cuda() for t in synthetic.make_inputs(w, "cpu"))
    dout = synthetic.make_dout(w, "cpu").cuda()
    out, lse = ring_attention(q, k, v, P, True, layout, w.scale)
    qs, ks, vs, outs, douts = (ring.split_shards(t, P, layout) for t in (q, k, v, out, dout))
    lses = [x.squeeze(-1).contiguous() for x in ring.split_shards(lse.unsqueeze(-1), P, layout)]
    vr = ring.VirtualBackwardRing(qs, ks, vs, outs, lses, douts, True, layout, w.scale)
    vr.run()
    torch.cuda.synchronize()
    first = [tuple(x.clone() for x in r) for r in vr.results()]
    got = [ring.join_shards([r[i] for r in first], layout) for i in range(3)]
    ref = oracle.attention_backward_reference(q.cpu(), k.cpu(), v.cpu(), dout.cpu(), True, w.scale)
    for name, g_, r_ in zip(("dq", "dk", "dv"), got, ref):
        assert_grad(g_, r_, f"virtual backward ring {layout} P={P} {name}")
    for ws in vr.ws:
        assert binding.ring_attn_status(ws.data_ptr(), torch.cuda.current_stream().cuda_stream) == 0
    vr.run(timing=True)
    torch.cuda.synchronize()
    for a, b in zip(first, vr.results()):
        assert all(torch.equal(x, y) for x, y in zip(a, b))
    # the caller's shards are untouched by the transfers
    for r in range(P):
        assert torch.equal(vr.k[r], ks[r]) and torch.equal(vr.v[r], vs[r])
