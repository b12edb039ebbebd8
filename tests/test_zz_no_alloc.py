"""GPU: ring_attn_fwd_noalloc, the forward whose scratch is the library's static device array.

Some callers cannot allocate device memory: a plain C host linking only this library,
or a serving process whose device memory is planned up front. This entry point takes
only inputs and outputs. Its results are checked against the fp64 oracle and against
ring_attn_fwd (the entry point with a caller workspace) on two calls in a row per
shape, since every call shares the one scratch array.

pytest collects this file last, so a run that stops at the first failure has already
run every other test. The tests pass in a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gpu_helpers import TOL, assert_parity
from sequence_exact_attention_ring_b200 import binding

pytestmark = pytest.mark.gpu

_LAYOUT = {"contiguous": binding.LAYOUT_CONTIGUOUS, "striped": binding.LAYOUT_STRIPED}


def _case(name, B, Hq, Hkv, S, D, P, causal, layout, seed):
    w = synthetic.custom(name, "bf16", B, Hq, Hkv, S, D, P, causal, layout, seed)
    q, k, v = (t.cuda() for t in synthetic.make_inputs(w, "cpu"))
    return w, q, k, v


def _args(w, q, k, v, out, lse):
    return (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), w.B, w.Hq, w.Hkv, w.S, w.D,
            w.P, int(w.causal), _LAYOUT[w.layout], w.scale, binding.DTYPE_BF16)


def test_noalloc_matches_oracle_and_workspace_entry_point_twice_in_a_row(cuda_lib):
    stream = torch.cuda.current_stream().cuda_stream
    cases = [_case("na1", 1, 4, 2, 2048, 128, 4, True, "striped", 31),
             _case("na2", 2, 2, 2, 1536, 64, 3, True, "contiguous", 32)]
    scratch_seen = set()
    t = TOL[torch.bfloat16]
    for w, q, k, v in cases:
        O_ref, L_ref = oracle.attention_reference(q.cpu(), k.cpu(), v.cpu(), w.causal, w.scale)
        # the existing entry point, with a workspace the test allocates
        out_ws = torch.empty_like(q)
        lse_ws = torch.empty((w.B, w.Hq, w.S), dtype=torch.float32, device="cuda")
        ws = torch.zeros(binding.ring_attn_fwd_workspace_bytes(w.B, w.Hq, w.Hkv, w.S, w.D, w.P, int(w.causal),
                                                               _LAYOUT[w.layout], binding.DTYPE_BF16),
                         dtype=torch.uint8, device="cuda")
        binding.check(binding.ring_attn_fwd(*_args(w, q, k, v, out_ws, lse_ws), ws.data_ptr(), ws.numel(), stream),
                      "ring_attn_fwd")
        assert binding.ring_attn_status(ws.data_ptr(), stream) == 0
        assert_parity(out_ws, lse_ws, O_ref, L_ref, torch.bfloat16, f"{w.name} ring_attn_fwd")

        for call in range(2):
            # outputs poisoned so a skipped write shows
            out = torch.full_like(q, float("nan"))
            lse = torch.full((w.B, w.Hq, w.S), float("nan"), dtype=torch.float32, device="cuda")
            torch.cuda.synchronize()
            free_before = torch.cuda.mem_get_info()[0]
            rc, scratch = binding.ring_attn_fwd_noalloc(*_args(w, q, k, v, out, lse), stream)
            binding.check(rc, "ring_attn_fwd_noalloc")
            assert scratch is not None and scratch % 256 == 0
            assert binding.ring_attn_status(scratch, stream) == 0
            if scratch in scratch_seen:
                # after the one-time setup no call takes device memory (seen by the driver,
                # not only by torch's caching allocator)
                assert torch.cuda.mem_get_info()[0] == free_before
            scratch_seen.add(scratch)
            assert_parity(out, lse, O_ref, L_ref, torch.bfloat16, f"{w.name} noalloc call {call}")
            assert (out.float() - out_ws.float()).abs().max().item() <= t["o_abs"]
            den = lse_ws.abs().clamp_min(1.0)
            assert ((lse - lse_ws).abs() / den).max().item() <= t["lse_rel"]
    assert len(scratch_seen) == 1  # one array per context, set up once


def test_noalloc_rejects_bad_arguments_without_launching(cuda_lib):
    stream = torch.cuda.current_stream().cuda_stream
    w, q, k, v = _case("na3", 1, 2, 2, 1024, 128, 4, True, "striped", 33)
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.S), dtype=torch.float32, device="cuda")
    a = list(_args(w, q, k, v, out, lse))
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")

    def both(args):
        """The no-allocation call and ring_attn_fwd return the same code for the same arguments."""
        rc = binding.ring_attn_fwd_noalloc(*args, stream)[0]
        assert rc == binding.ring_attn_fwd(*args, ws.data_ptr(), ws.numel(), stream)
        return rc

    bad_s = list(a)
    bad_s[8] = 1022  # S % P != 0 (P = 4)
    assert both(bad_s) == binding.EINVAL
    bad_d = list(a)
    bad_d[9] = 96  # head dim outside {64, 128}
    assert both(bad_d) == binding.EUNSUPPORTED
    bad_scale = list(a)
    bad_scale[13] = -1.0
    assert both(bad_scale) == binding.EINVAL
    bad_align = list(a)
    bad_align[3] = out.data_ptr() + 2
    assert both(bad_align) == binding.EALIGN
    rc, scratch = binding.ring_attn_fwd_noalloc(*a, stream)
    assert rc == binding.OK and binding.ring_attn_status(scratch, stream) == 0
    O_ref, L_ref = oracle.attention_reference(q.cpu(), k.cpu(), v.cpu(), w.causal, w.scale)
    assert_parity(out, lse, O_ref, L_ref, torch.bfloat16, "noalloc after rejected calls")
    assert np.isfinite(lse.cpu().numpy()).all()
