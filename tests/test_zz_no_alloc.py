"""GPU: ring_attn_fwd_noalloc (scratch in the library's static device array) against ring_attn_fwd.

Collected last on purpose: it must pass in a fresh process and after every other test.
"""
import pytest
import torch

import synthetic
from gpu_helpers import TOL
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


def test_noalloc_matches_workspace_entry_point_twice_in_a_row(cuda_lib):
    stream = torch.cuda.current_stream().cuda_stream
    cases = [_case("na1", 1, 4, 2, 2048, 128, 4, True, "striped", 31),
             _case("na2", 2, 2, 2, 1536, 64, 3, True, "contiguous", 32)]
    scratch_seen = set()
    for w, q, k, v in cases:
        # the existing entry point, with a workspace the test allocates
        out_ref = torch.empty_like(q)
        lse_ref = torch.empty((w.B, w.Hq, w.S), dtype=torch.float32, device="cuda")
        ws = torch.zeros(binding.ring_attn_fwd_workspace_bytes(w.B, w.Hq, w.Hkv, w.S, w.D, w.P, int(w.causal),
                                                               _LAYOUT[w.layout], binding.DTYPE_BF16),
                         dtype=torch.uint8, device="cuda")
        binding.check(binding.ring_attn_fwd(*_args(w, q, k, v, out_ref, lse_ref), ws.data_ptr(), ws.numel(), stream),
                      "ring_attn_fwd")
        assert binding.ring_attn_status(ws.data_ptr(), stream) == 0

        # the no-allocation entry point: outputs poisoned so a skipped write shows
        out = torch.full_like(q, float("nan"))
        lse = torch.full((w.B, w.Hq, w.S), float("nan"), dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
        before = torch.cuda.memory_allocated()
        rc, scratch = binding.ring_attn_fwd_noalloc(*_args(w, q, k, v, out, lse), stream)
        binding.check(rc, "ring_attn_fwd_noalloc")
        assert scratch is not None and scratch % 256 == 0
        assert binding.ring_attn_status(scratch, stream) == 0
        assert torch.cuda.memory_allocated() == before
        scratch_seen.add(scratch)

        t = TOL[torch.bfloat16]
        assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
        assert (out.float() - out_ref.float()).abs().max().item() <= t["o_abs"]
        den = lse_ref.abs().clamp_min(1.0)
        assert ((lse - lse_ref).abs() / den).max().item() <= t["lse_rel"]
    assert len(scratch_seen) == 1  # one array per device, set up once


def test_noalloc_rejects_bad_arguments_without_launching(cuda_lib):
    stream = torch.cuda.current_stream().cuda_stream
    w, q, k, v = _case("na3", 1, 2, 2, 1024, 128, 4, True, "striped", 33)
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.S), dtype=torch.float32, device="cuda")
    a = list(_args(w, q, k, v, out, lse))
    bad_s = list(a)
    bad_s[8] = 1022  # S % P != 0 (P = 4)
    assert binding.ring_attn_fwd_noalloc(*bad_s, stream)[0] == binding.EINVAL
    bad_scale = list(a)
    bad_scale[13] = -1.0
    assert binding.ring_attn_fwd_noalloc(*bad_scale, stream)[0] == binding.EINVAL
    bad_align = list(a)
    bad_align[3] = out.data_ptr() + 2
    assert binding.ring_attn_fwd_noalloc(*bad_align, stream)[0] == binding.EALIGN
    rc, scratch = binding.ring_attn_fwd_noalloc(*a, stream)
    assert rc == binding.OK and binding.ring_attn_status(scratch, stream) == 0
