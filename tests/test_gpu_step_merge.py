"""GPU: the literal ring step, the merge kernel, and the bounded-wait status path."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gpu_helpers import assert_parity
from sequence_exact_attention_ring_b200 import binding, merge, ring_attention, ring_attention_step

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("algo,dtype", [("tcgen05", "bf16"), ("tcgen05_1sm", "bf16"), ("simt", "bf16"),
                                        ("simt", "fp32")])
@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
def test_ring_steps_merged_equal_full_forward(cuda_lib, algo, dtype, layout):
    """Device i's P ring steps (one literal block each), merged, give the fused result."""
    B, Hq, Hkv, D, P = 1, 2, 2, 128, 4
    S = 2048 if layout == "zigzag" else 1152
    w = synthetic.custom("steps", dtype, B, Hq, Hkv, S, D, P, True, layout, 5)
    q, k, v = (t.cuda() for t in synthetic.make_inputs(w, "cpu"))
    O_ref, L_ref = oracle.attention_reference(q.cpu(), k.cpu(), v.cpu(), True, w.scale)
    for i in range(P):
        parts = [ring_attention_step(q, k, v, P, i, (i - s) % P, True, layout, w.scale, algo=algo)
                 for s in range(P)]
        o_parts = torch.stack([p[0] for p in parts]).contiguous()
        l_parts = torch.stack([p[1] for p in parts]).contiguous()
        o, l = merge(o_parts, l_parts, torch.float32)
        torch.cuda.synchronize()
        toks = oracle.shard_tokens(S, P, layout, i)
        tol_dtype = torch.float32 if dtype == "fp32" else torch.bfloat16
        assert_parity(o, l, O_ref[:, :, toks], L_ref[:, :, toks], tol_dtype, f"shard {i}")


def test_step_block_matches_oracle_keyset(cuda_lib):
    """A single step against the oracle restricted to that block's allowed keys (empty rows -> -inf)."""
    B, Hq, Hkv, S, D, P = 1, 2, 2, 512, 64, 4
    w = synthetic.custom("blk", "bf16", B, Hq, Hkv, S, D, P, True, "striped", 9)
    q, k, v = (t.cuda() for t in synthetic.make_inputs(w, "cpu"))
    i, j = 1, 3  # j > i under striped causal: the diagonal key is excluded, row 0 is empty
    o, l = ring_attention_step(q, k, v, P, i, j, True, "striped", w.scale)
    torch.cuda.synchronize()
    tq = oracle.shard_tokens(S, P, "striped", i)
    tk = oracle.shard_tokens(S, P, "striped", j)
    mask = np.zeros((B, Hq, S, S), dtype=bool)
    mask[:, :, tq[:, None], tk[None, :]] = oracle.block_allowed(tq, tk, True)
    O_ref, L_ref = oracle.attention_keyset(q.cpu(), k.cpu(), v.cpu(), mask, w.scale)
    O_ref, L_ref = O_ref[:, :, tq], L_ref[:, :, tq]
    assert torch.isneginf(l[:, :, 0]).all()
    assert (o[:, :, 0] == 0).all()
    fin = np.isfinite(L_ref)
    assert (torch.isneginf(l).cpu().numpy() == ~fin).all()
    lo, ll = o.cpu().numpy(), l.cpu().numpy()
    assert np.abs(lo[fin] - O_ref[fin]).max() <= 2e-2
    assert (np.abs(ll[fin] - L_ref[fin]) / np.maximum(np.abs(L_ref[fin]), 1)).max() <= 1e-3


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_merge_kernel_against_oracle(cuda_lib, out_dtype):
    g = torch.Generator().manual_seed(11)
    n, rows, D = 5, 3000, 128
    o = torch.randn((n, rows, D), generator=g)
    l = torch.randn((n, rows), generator=g) * 4
    l[1, ::3] = -torch.inf            # empty parts
    l[:, 7] = -torch.inf              # an all-empty row
    O_ref, L_ref = oracle.merge_partials(list(o.numpy()), list(l.numpy()))
    out, lse = merge(o.cuda(), l.cuda(), out_dtype)
    torch.cuda.synchronize()
    tol = 1e-5 if out_dtype == torch.float32 else 2e-2
    got = out.float().cpu().numpy()
    assert np.abs(got - O_ref).max() <= tol
    fin = np.isfinite(L_ref)
    assert np.isneginf(lse.cpu().numpy()[~fin]).all() and (got[~fin] == 0).all()
    assert np.abs(lse.cpu().numpy()[fin] - L_ref[fin]).max() <= 1e-5


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("n,rows,D", [(320, 8, 128), (37, 5, 64), (1024, 3, 128)])
def test_merge_many_parts_few_rows(cuda_lib, out_dtype, n, rows, D):
    """The decode-shaped merge (one block per row, parts split across its threads)."""
    g = torch.Generator().manual_seed(12 + n)
    o = torch.randn((n, rows, D), generator=g)
    l = torch.randn((n, rows), generator=g) * 6
    l[::7, 0] = -torch.inf            # scattered empty parts
    l[:, rows - 1] = -torch.inf       # an all-empty row
    O_ref, L_ref = oracle.merge_partials(list(o.numpy()), list(l.numpy()))
    out, lse = merge(o.cuda(), l.cuda(), out_dtype)
    torch.cuda.synchronize()
    tol = 1e-5 if out_dtype == torch.float32 else 2e-2
    got = out.float().cpu().numpy()
    assert np.abs(got - O_ref).max() <= tol
    fin = np.isfinite(L_ref)
    assert np.isneginf(lse.cpu().numpy()[~fin]).all() and (got[~fin] == 0).all()
    assert np.abs(lse.cpu().numpy()[fin] - L_ref[fin]).max() <= 1e-5


def test_watchdog_gives_up_and_context_stays_usable(cuda_lib):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert binding.ring_attn_debug_watchdog(50_000, ws.data_ptr(), 256, s) == 0
    assert binding.ring_attn_status(ws.data_ptr(), s) == binding.ETIMEOUT
    # a normal call afterwards succeeds and resets the status word
    w = synthetic.custom("after", "bf16", 1, 2, 2, 512, 128, 4, True, "striped", 1)
    q, k, v = (t.cuda() for t in synthetic.make_inputs(w, "cpu"))
    out, lse = ring_attention(q, k, v, 4, True, "striped", workspace=ws)
    assert binding.ring_attn_status(ws.data_ptr(), s) == 0
    O_ref, L_ref = oracle.attention_reference(q.cpu(), k.cpu(), v.cpu(), True, w.scale)
    assert_parity(out, lse, O_ref, L_ref, torch.bfloat16, "after watchdog")


def test_host_runner_end_to_end(cuda_lib):
    from sequence_exact_attention_ring_b200 import HostRunner
    w = synthetic.custom("e2e", "bf16", 1, 4, 2, 2048, 128, 8, True, "striped", 21)
    q, k, v = synthetic.make_inputs(w, "cpu")
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    r = HostRunner(q.shape, k.shape, torch.bfloat16, w.P, True, "striped", w.scale)
    out, lse = r.run(qh, kh, vh)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle.attention_reference(q, k, v, True, w.scale)
    assert_parity(out, lse, O_ref, L_ref, torch.bfloat16, "host runner")


def test_host_runner_pipelined_steps(cuda_lib):
    """Three different inputs through two buffer sets and two streams: each step's host
    result is the oracle's for its own inputs."""
    from sequence_exact_attention_ring_b200 import HostRunner
    ws = [synthetic.custom("e2e", "bf16", 1, 4, 2, 1024, 128, 4, True, "striped", 31 + n) for n in range(3)]
    inputs = [tuple(t.pin_memory() for t in synthetic.make_inputs(w, "cpu")) for w in ws]
    r = HostRunner(inputs[0][0].shape, inputs[0][1].shape, torch.bfloat16, 4, True, "striped", ws[0].scale,
                   buffers=2)
    copy_stream, compute_stream = torch.cuda.Stream(), torch.cuda.Stream()
    results = []
    for n in range(3):  # one step at a time, keeping each result before its set is reused
        out, lse = r.run_steps([inputs[n]], copy_stream, compute_stream)
        copy_stream.synchronize()
        results.append((out.clone(), lse.clone()))
    out, lse = r.run_steps(inputs, copy_stream, compute_stream)  # all three pipelined
    copy_stream.synchronize()
    results.append((out.clone(), lse.clone()))
    for n, (o, l) in enumerate(results):
        q, k, v = inputs[min(n, 2)]
        O_ref, L_ref = oracle.attention_reference(q, k, v, True, ws[0].scale)
        assert_parity(o, l, O_ref, L_ref, torch.bfloat16, f"pipelined step {n}")
