"""Torch-facing calls over the C ABI. PyTorch supplies device memory and streams.

Marshalling only: shapes/dtypes are checked, buffers allocated with torch, and the
library's kernels do every step of the computation.
"""
from __future__ import annotations

import math

import torch

from . import binding as _b

_LAYOUTS = {"contiguous": _b.LAYOUT_CONTIGUOUS, "striped": _b.LAYOUT_STRIPED, "zigzag": _b.LAYOUT_ZIGZAG}
_ALGOS = {"auto": _b.ALGO_AUTO, "simt": _b.ALGO_SIMT, "tcgen05": _b.ALGO_TCGEN05,
          "tcgen05_1sm": _b.ALGO_TCGEN05_1SM}
_DTYPES = {torch.float32: _b.DTYPE_FP32, torch.bfloat16: _b.DTYPE_BF16}


def _stream_ptr(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _layout(layout) -> int:
    return _LAYOUTS[layout] if isinstance(layout, str) else int(layout)


def _check_qkv(q, k, v):
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [B, H, S, D]")
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("q, k, v must be CUDA tensors (use ring_attention_host for host buffers)")
    if q.dtype not in _DTYPES or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share dtype float32 or bfloat16")
    if k.shape != v.shape or q.shape[0] != k.shape[0] or q.shape[2:] != k.shape[2:]:
        raise ValueError("shape mismatch: q [B,Hq,S,D], k/v [B,Hkv,S,D]")
    if not (q.is_contiguous() and k.is_contiguous() and v.is_contiguous()):
        raise ValueError("q, k, v must be contiguous")


def workspace_bytes(q: torch.Tensor, k: torch.Tensor, P: int, causal: bool, layout) -> int:
    B, Hq, S, D = q.shape
    n = _b.ring_attn_fwd_workspace_bytes(B, Hq, k.shape[1], S, D, P, int(causal), _layout(layout),
                                         _DTYPES[q.dtype])
    if n == 0:
        raise _b.RingAttnError(_b.EINVAL, "ring_attn_fwd_workspace_bytes")
    return n


def ring_attention(q, k, v, P: int, causal: bool = True, layout="striped", scale: float | None = None,
                   algo: str = "auto", out=None, lse=None, workspace=None, stream=None):
    """Exact attention of q [B,Hq,S,D] over k/v [B,Hkv,S,D] folded in P ring shards.

    Returns (out [B,Hq,S,D] in q's dtype, lse [B,Hq,S] fp32). Asynchronous on `stream`.
    """
    _check_qkv(q, k, v)
    B, Hq, S, D = q.shape
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, S), dtype=torch.float32, device=q.device)
    wsb = workspace_bytes(q, k, P, causal, layout)
    if workspace is None:
        workspace = torch.empty(wsb, dtype=torch.uint8, device=q.device)
    rc = _b.ring_attn_fwd_algo(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                               B, Hq, k.shape[1], S, D, P, int(causal), _layout(layout), scale,
                               _DTYPES[q.dtype], workspace.data_ptr(), workspace.numel(), _stream_ptr(stream),
                               _ALGOS[algo])
    _b.check(rc, "ring_attn_fwd")
    return out, lse


def ring_attention_step(q, k, v, P: int, q_shard: int, kv_shard: int, causal: bool = True, layout="striped",
                        scale: float | None = None, algo: str = "auto", stream=None):
    """One ring step: normalised partial (o [B,Hq,Sq,D] fp32, lse [B,Hq,Sq]) in shard-local order."""
    _check_qkv(q, k, v)
    B, Hq, S, D = q.shape
    Sq = S // P
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    o = torch.empty((B, Hq, Sq, D), dtype=torch.float32, device=q.device)
    lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    wsb = workspace_bytes(q, k, P, causal, layout)
    ws = torch.empty(wsb, dtype=torch.uint8, device=q.device)
    rc = _b.ring_attn_fwd_step(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq,
                               k.shape[1], S, D, P, q_shard, kv_shard, int(causal), _layout(layout), scale,
                               _DTYPES[q.dtype], _ALGOS[algo], ws.data_ptr(), ws.numel(), _stream_ptr(stream))
    _b.check(rc, "ring_attn_fwd_step")
    return o, lse


def ring_attention_ring_step(q_shard, k_shard, v_shard, S: int, P: int, q_index: int, kv_index: int,
                             causal: bool = True, layout="striped", scale: float | None = None, first: bool = False,
                             last: bool = False, o_acc=None, lse_acc=None, out=None, lse_out=None, workspace=None,
                             stream=None):
    """One ring step on shard-local buffers (as one device of a multi-device ring runs it).

    q_shard [B,Hq,Sq,D] is query shard q_index and k_shard/v_shard [B,Hkv,Sq,D] KV shard
    kv_index, each in shard-local order. The step's block result is folded into the
    running state o_acc [B,Hq,Sq,D] fp32 / lse_acc [B,Hq,Sq] (started on `first`); on
    `last` the merged rows go to out (q's dtype) and lse_out. Returns (out, lse_out) on
    a last step, else (o_acc, lse_acc). Asynchronous on `stream`.
    """
    _check_qkv(q_shard, k_shard, v_shard)
    B, Hq, Sq, D = q_shard.shape
    if Sq * P != S:
        raise ValueError("shards must hold S / P rows")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dev = q_shard.device
    if not (first and last):
        for t, shape in ((o_acc, (B, Hq, Sq, D)), (lse_acc, (B, Hq, Sq))):
            if t is None or tuple(t.shape) != shape or t.dtype != torch.float32 or not t.is_contiguous():
                raise ValueError("o_acc [B,Hq,Sq,D] and lse_acc [B,Hq,Sq] must be contiguous float32 tensors")
    if last:
        if out is None:
            out = torch.empty_like(q_shard)
        if lse_out is None:
            lse_out = torch.empty((B, Hq, Sq), dtype=torch.float32, device=dev)
    if workspace is None:
        wsb = _b.ring_attn_fwd_workspace_bytes(B, Hq, k_shard.shape[1], S, D, P, int(causal), _layout(layout),
                                               _DTYPES[q_shard.dtype])
        if wsb == 0:
            raise _b.RingAttnError(_b.EINVAL, "ring_attn_fwd_workspace_bytes")
        workspace = torch.empty(wsb, dtype=torch.uint8, device=dev)
    flags = (_b.STEP_FIRST if first else 0) | (_b.STEP_LAST if last else 0)
    ptr = lambda t: 0 if t is None else t.data_ptr()  # noqa: E731
    rc = _b.ring_attn_fwd_ring_step(q_shard.data_ptr(), k_shard.data_ptr(), v_shard.data_ptr(), ptr(o_acc),
                                    ptr(lse_acc), ptr(out), ptr(lse_out), B, Hq, k_shard.shape[1], S, D, P, q_index,
                                    kv_index, int(causal), _layout(layout), scale, _DTYPES[q_shard.dtype], flags,
                                    workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
    _b.check(rc, "ring_attn_fwd_ring_step")
    return (out, lse_out) if last else (o_acc, lse_acc)


def ring_attention_backward(q, k, v, out, lse, dout, P: int, causal: bool = True, layout="striped",
                            scale: float | None = None, workspace=None, stream=None):
    """Gradients (dq, dk, dv) of ring_attention's output against dout, from its out and lse.

    bf16 tensors, D = 128. Asynchronous on `stream`.
    """
    _check_qkv(q, k, v)
    for t, name in ((out, "out"), (dout, "dout")):
        if t.shape != q.shape or t.dtype != q.dtype or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor shaped and typed like q")
    B, Hq, S, D = q.shape
    if lse.shape != (B, Hq, S) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [B, Hq, S] tensor")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    wsb = _b.ring_attn_bwd_workspace_bytes(B, Hq, k.shape[1], S, D, P, int(causal), _layout(layout),
                                           _DTYPES[q.dtype])
    if wsb == 0:
        raise _b.RingAttnError(_b.EINVAL, "ring_attn_bwd_workspace_bytes")
    if workspace is None or workspace.numel() < wsb:
        workspace = torch.empty(wsb, dtype=torch.uint8, device=q.device)
    rc = _b.ring_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), dout.data_ptr(),
                          dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, k.shape[1], S, D, P, int(causal),
                          _layout(layout), scale, _DTYPES[q.dtype], workspace.data_ptr(), workspace.numel(),
                          _stream_ptr(stream))
    _b.check(rc, "ring_attn_bwd")
    return dq, dk, dv


def _ptr(t) -> int:
    return 0 if t is None else t.data_ptr()


def ring_backward_prep(out_shard, lse_shard, dout_shard, S: int, P: int, q_index: int, causal: bool = True,
                       layout="striped", workspace=None, stream=None):
    """Row statistics of query shard q_index for a backward pass spread over a ring of devices.

    out_shard, dout_shard [B,Hq,Sq,D] bf16 and lse_shard [B,Hq,Sq] fp32 in shard-local order
    (as ring_attention_ring_step wrote them). Returns the workspace that every
    ring_backward_step of this pass then uses. Asynchronous on `stream`.
    """
    B, Hq, Sq, D = out_shard.shape
    if Sq * P != S:
        raise ValueError("shards must hold S / P rows")
    for t in (out_shard, dout_shard):
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.shape != out_shard.shape:
            raise ValueError("out_shard and dout_shard must be contiguous bf16 CUDA tensors of one shape")
    if lse_shard.shape != (B, Hq, Sq) or lse_shard.dtype != torch.float32 or not lse_shard.is_contiguous():
        raise ValueError("lse_shard must be a contiguous float32 [B, Hq, Sq] tensor")
    # the key-value head count does not change the statistics' size; use Hq
    wsb = _b.ring_attn_bwd_ring_workspace_bytes(B, Hq, Hq, S, D, P, int(causal), _layout(layout), _b.DTYPE_BF16)
    if wsb == 0:
        raise _b.RingAttnError(_b.EINVAL, "ring_attn_bwd_ring_workspace_bytes")
    if workspace is None or workspace.numel() < wsb:
        workspace = torch.empty(wsb, dtype=torch.uint8, device=out_shard.device)
    rc = _b.ring_attn_bwd_ring_prep(out_shard.data_ptr(), lse_shard.data_ptr(), dout_shard.data_ptr(), B, Hq, Hq, S, D,
                                    P, q_index, int(causal), _layout(layout), _b.DTYPE_BF16, workspace.data_ptr(),
                                    workspace.numel(), _stream_ptr(stream))
    _b.check(rc, "ring_attn_bwd_ring_prep")
    return workspace


def ring_backward_step(q_shard, dout_shard, k_shard, v_shard, S: int, P: int, q_index: int, kv_index: int,
                       workspace, causal: bool = True, layout="striped", scale: float | None = None, parts=3,
                       first: bool = False, last: bool = False, dq_acc=None, dk_acc=None, dv_acc=None, dq=None,
                       dk=None, dv=None, stream=None):
    """One step of the backward ring: the dK/dV contributions of query shard q_index to KV
    shard kv_index (parts & 1, folded into dk_acc/dv_acc) and/or the dQ contribution of KV
    shard kv_index to query shard q_index (parts & 2, folded into dq_acc). Accumulators are
    fp32, started on `first`; on `last` the bf16 gradients are written to dq / dk, dv.
    All tensors are single shards in shard-local order. Asynchronous on `stream`."""
    _check_qkv(q_shard, k_shard, v_shard)
    B, Hq, Sq, D = q_shard.shape
    if Sq * P != S:
        raise ValueError("shards must hold S / P rows")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    flags = (_b.STEP_FIRST if first else 0) | (_b.STEP_LAST if last else 0)
    rc = _b.ring_attn_bwd_ring_step(q_shard.data_ptr(), dout_shard.data_ptr(), k_shard.data_ptr(), v_shard.data_ptr(),
                                    _ptr(dq_acc), _ptr(dk_acc), _ptr(dv_acc), _ptr(dq), _ptr(dk), _ptr(dv), B, Hq,
                                    k_shard.shape[1], S, D, P, q_index, kv_index, int(causal), _layout(layout), scale,
                                    _DTYPES[q_shard.dtype], int(parts), flags, workspace.data_ptr(),
                                    workspace.numel(), _stream_ptr(stream))
    _b.check(rc, "ring_attn_bwd_ring_step")


def ring_attention_decode(q1, k, v, P: int, layout="striped", scale: float | None = None, workspace=None,
                          stream=None):
    """One decode step: q1 [B, Hq, D] (one new row per head) against the cache k, v [B, Hkv, S, D]
    kept in P ring shards. Returns (out [B, Hq, D] bf16, lse [B, Hq] fp32). Asynchronous on `stream`."""
    if q1.dim() != 3 or k.dim() != 4 or v.shape != k.shape:
        raise ValueError("q1 must be [B, Hq, D] and k, v [B, Hkv, S, D]")
    for t in (q1, k, v):
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("q1, k, v must be contiguous bf16 CUDA tensors")
    B, Hq, D = q1.shape
    Hkv, S = k.shape[1], k.shape[2]
    if k.shape[0] != B or k.shape[3] != D:
        raise ValueError("shape mismatch between q1 and the cache")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    out = torch.empty_like(q1)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q1.device)
    wsb = _b.ring_attn_decode_workspace_bytes(B, Hq, Hkv, S, D, P, _layout(layout), _b.DTYPE_BF16)
    if wsb == 0:
        raise _b.RingAttnError(_b.EINVAL, "ring_attn_decode_workspace_bytes")
    if workspace is None or workspace.numel() < wsb:
        workspace = torch.empty(wsb, dtype=torch.uint8, device=q1.device)
    rc = _b.ring_attn_decode(q1.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, S,
                             D, P, _layout(layout), scale, _b.DTYPE_BF16, workspace.data_ptr(), workspace.numel(),
                             _stream_ptr(stream))
    _b.check(rc, "ring_attn_decode")
    return out, lse


def merge(o_parts: torch.Tensor, lse_parts: torch.Tensor, out_dtype=torch.float32, stream=None):
    """Merge normalised partials o_parts [n, ..., D] fp32 / lse_parts [n, ...] -> (out [..., D], lse [...])."""
    if o_parts.dtype != torch.float32 or lse_parts.dtype != torch.float32:
        raise ValueError("partials must be float32")
    if not (o_parts.is_cuda and lse_parts.is_cuda and o_parts.is_contiguous() and lse_parts.is_contiguous()):
        raise ValueError("partials must be contiguous CUDA tensors")
    n, D = o_parts.shape[0], o_parts.shape[-1]
    lead = o_parts.shape[1:-1]
    if tuple(lse_parts.shape) != (n, *lead):
        raise ValueError("lse_parts must be [n, ...] matching o_parts [n, ..., D]")
    rows = int(math.prod(lead))
    out = torch.empty((*lead, D), dtype=out_dtype, device=o_parts.device)
    lse = torch.empty(lead, dtype=torch.float32, device=o_parts.device)
    rc = _b.ring_attn_merge(o_parts.data_ptr(), lse_parts.data_ptr(), n, rows, D, out.data_ptr(), lse.data_ptr(),
                            _DTYPES[out_dtype], _stream_ptr(stream))
    _b.check(rc, "ring_attn_merge")
    return out, lse


def status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise and return the workspace status word (0 or binding.ETIMEOUT)."""
    return _b.ring_attn_status(workspace.data_ptr(), _stream_ptr(stream))


class HostRunner:
    """End-to-end path for host-resident inputs: pinned host -> device copies,
    ring_attn_fwd, device -> pinned host copies.

    Device buffers are allocated once (by torch) and reused across calls. `run` does
    one step on one stream. `run_steps` runs many steps as a pipeline over `buffers`
    device buffer sets and two streams: the copies of one step overlap the kernel of
    another, as a serving loop would run them.
    """

    def __init__(self, shape_q, shape_kv, dtype, P, causal=True, layout="striped", scale=None, device="cuda",
                 buffers=1):
        self.P, self.causal, self.layout = P, causal, layout
        B, Hq, S, D = shape_q
        self.scale = 1.0 / math.sqrt(D) if scale is None else scale
        self.sets = []
        for _ in range(max(1, buffers)):
            st = {
                "q": torch.empty(shape_q, dtype=dtype, device=device),
                "k": torch.empty(shape_kv, dtype=dtype, device=device),
                "v": torch.empty(shape_kv, dtype=dtype, device=device),
                "out": torch.empty(shape_q, dtype=dtype, device=device),
                "lse": torch.empty((B, Hq, S), dtype=torch.float32, device=device),
                "out_host": torch.empty(shape_q, dtype=dtype, pin_memory=True),
                "lse_host": torch.empty((B, Hq, S), dtype=torch.float32, pin_memory=True),
            }
            st["ws"] = torch.empty(workspace_bytes(st["q"], st["k"], P, causal, layout), dtype=torch.uint8,
                                   device=device)
            self.sets.append(st)
        first = self.sets[0]
        self.q, self.k, self.v, self.out, self.lse = first["q"], first["k"], first["v"], first["out"], first["lse"]
        self.out_host, self.lse_host, self.ws = first["out_host"], first["lse_host"], first["ws"]

    def h2d_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.q, self.k, self.v))

    def d2h_bytes(self) -> int:
        return self.out.numel() * self.out.element_size() + self.lse.numel() * 4

    def _forward(self, st, stream):
        ring_attention(st["q"], st["k"], st["v"], self.P, self.causal, self.layout, self.scale, out=st["out"],
                       lse=st["lse"], workspace=st["ws"], stream=stream)

    def run(self, q_host, k_host, v_host, stream=None):
        s = stream if stream is not None else torch.cuda.current_stream()
        st = self.sets[0]
        with torch.cuda.stream(s):
            st["q"].copy_(q_host, non_blocking=True)
            st["k"].copy_(k_host, non_blocking=True)
            st["v"].copy_(v_host, non_blocking=True)
            self._forward(st, s)
            st["out_host"].copy_(st["out"], non_blocking=True)
            st["lse_host"].copy_(st["lse"], non_blocking=True)
        return st["out_host"], st["lse_host"]

    def run_steps(self, batches, copy_stream, compute_stream):
        """Pipelined steps over the buffer sets: every (q_host, k_host, v_host) in `batches`
        is copied in on `copy_stream`, folded on `compute_stream` once its copy landed,
        and its out and lse copied back on `copy_stream` once the kernel finished. Step n
        uses set n % buffers; its host results stay valid until step n + buffers starts.
        Asynchronous: synchronize copy_stream to wait for everything."""
        nb = len(self.sets)
        batches = list(batches)
        h2d_done = [torch.cuda.Event() for _ in batches]
        fwd_done = [torch.cuda.Event() for _ in batches]

        def h2d(n):
            st = self.sets[n % nb]
            qh, kh, vh = batches[n]
            with torch.cuda.stream(copy_stream):
                st["q"].copy_(qh, non_blocking=True)
                st["k"].copy_(kh, non_blocking=True)
                st["v"].copy_(vh, non_blocking=True)
                h2d_done[n].record(copy_stream)

        def d2h(n):
            st = self.sets[n % nb]
            copy_stream.wait_event(fwd_done[n])
            with torch.cuda.stream(copy_stream):
                st["out_host"].copy_(st["out"], non_blocking=True)
                st["lse_host"].copy_(st["lse"], non_blocking=True)

        # copy stream order: H2D of the first `nb` steps, then for each step its D2H
        # followed by the H2D of the step that reuses its buffer set
        for n in range(min(nb, len(batches))):
            h2d(n)
        for n in range(len(batches)):
            compute_stream.wait_event(h2d_done[n])
            self._forward(self.sets[n % nb], compute_stream)
            fwd_done[n].record(compute_stream)
            d2h(n)
            if n + nb < len(batches):
                h2d(n + nb)
        last = self.sets[(len(batches) - 1) % nb]
        return last["out_host"], last["lse_host"]
