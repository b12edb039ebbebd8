"""Exact ring attention spread over ranks: each rank keeps one query shard while the
KV shards travel around the ring.

RingAttention deep-architecture article (techknowgenie):
  * section 2 "core principle": with N ranks, rank r keeps query shard r; after each
    step the KV block it holds moves on to rank (r + 1) mod N and the block of rank
    (r - 1) mod N arrives, so at step s rank r holds KV shard (r - s) mod N.
  * section 4 "zero-bubble condition": the next block's transfer hides behind the
    current block's compute when T_comm <= T_compute (2*2*Sq*D bytes of K and V per
    head against 4*Sq^2*D FLOPs per block step).
  * section 5 listing: a current and a next KV buffer, the sends and receives issued
    on their own stream, a wait before the swap, and the fold of every block into the
    running (m, l, O) state, with the output produced after the last step.
  * section "activation checkpointing and memory recomputation": in the backward pass
    the KV blocks travel the ring the other way, so rank r holds KV shard (r + s) mod N
    at step s (direction -1 of ring_steps and run_ring_pass).

Every step's attention arithmetic is one ring_attn_fwd_ring_step call: the fused
kernel, whose epilogue folds the block into the running state. This module only
orders the transfers and the calls on streams; it moves bytes and never computes
attention.

Two transports carry the KV shards:
  * processes, one per GPU, over torch.distributed point-to-point sends and receives
    (NCCL over NVLink between GPUs; gloo on the host for the bookkeeping tests). The
    received shard lands in this GPU's own memory and the kernel loads it from there;
  * virtual ranks inside one process, each with its own buffers and streams on one
    device: a device-to-device copy on the rank's copy stream pulls the previous rank's
    current shard into this rank's next buffer while its compute stream runs the step.
    No kernel of one rank waits on another rank's kernel; streams are ordered by events.
"""
from __future__ import annotations

import contextlib
import math
from typing import NamedTuple

import torch

from .api import ring_attention_ring_step

_LAYOUTS = ("contiguous", "striped", "zigzag")


# ------------------------------------------------------------------ schedule

def ring_steps(rank: int, world: int, direction: int = 1):
    """The steps of one rank: (step s, KV shard held, rank sent to, rank received from).

    direction +1 is the forward ring (shard (rank - s) mod world at step s, blocks move to
    rank + 1); -1 the backward ring (shard (rank + s) mod world, blocks move to rank - 1).
    """
    if direction not in (1, -1):
        raise ValueError("direction must be +1 or -1")
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    return [(s, (rank - direction * s) % world, (rank + direction) % world, (rank - direction) % world)
            for s in range(world)]


# ------------------------------------------------------------------ shard layout helpers

def shard_token_index(S: int, P: int, layout: str, i: int) -> torch.Tensor:
    """Global tokens of shard i in shard-local order (contiguous: [i*Sq, (i+1)*Sq);
    striped: a*P + i; zigzag: chunks i and 2P-1-i of C = S/(2P) tokens)."""
    if layout not in _LAYOUTS or S % P or (layout == "zigzag" and S % (2 * P)):
        raise ValueError("bad shard geometry")
    Sq = S // P
    a = torch.arange(Sq, dtype=torch.int64)
    if layout == "contiguous":
        return i * Sq + a
    if layout == "striped":
        return a * P + i
    C = Sq // 2
    return torch.where(a < C, i * C + a, (2 * P - 1 - i) * C + (a - C))


def split_shards(x: torch.Tensor, P: int, layout: str):
    """[B, H, S, D] in token order -> P contiguous [B, H, Sq, D] shards in shard-local order
    (input preparation for the ring; each rank of a real ring already holds its shard)."""
    S = x.shape[2]
    return [x.index_select(2, shard_token_index(S, P, layout, i).to(x.device)).contiguous() for i in range(P)]


def join_shards(shards, layout: str) -> torch.Tensor:
    """Inverse of split_shards: P shards [B, H, Sq, ...] -> [B, H, S, ...] in token order."""
    P = len(shards)
    Sq = shards[0].shape[2]
    S = P * Sq
    full = torch.empty((*shards[0].shape[:2], S, *shards[0].shape[3:]), dtype=shards[0].dtype,
                       device=shards[0].device)
    for i, sh in enumerate(shards):
        full.index_copy_(2, shard_token_index(S, P, layout, i).to(sh.device), sh)
    return full


# ------------------------------------------------------------------ one rank per process

def run_ring_pass(k_shard: torch.Tensor, v_shard: torch.Tensor, step_fn, group=None, direction: int = 1,
                  compute_stream=None, comm_stream=None):
    """Runs the world_size steps of this rank, passing the (K, V) pair around the ring.

    step_fn(s, kv_index, k_cur, v_cur, first, last) issues step s on the compute stream
    (the current stream while it runs). Between steps the pair held now is sent to the
    next rank and the previous rank's pair received into the other buffer, on
    comm_stream, while step s runs; step s + 1 waits for that transfer. A receive into a
    buffer waits until the step that read it (two steps earlier) has finished. Every rank
    takes the same collective steps in the same order. CUDA tensors go through NCCL
    with streams; CPU tensors (gloo) run the same order synchronously.
    """
    import torch.distributed as dist

    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    cuda = k_shard.is_cuda
    if cuda:
        compute_stream = compute_stream or torch.cuda.current_stream(k_shard.device)
        comm_stream = comm_stream or torch.cuda.Stream(k_shard.device)
        comm_stream.wait_stream(compute_stream)  # the inputs are ready where the caller made them
    bufs = [(torch.empty_like(k_shard), torch.empty_like(v_shard)) for _ in range(2 if world > 1 else 0)]
    peer = (lambda r: dist.get_global_rank(group, r)) if group is not None else (lambda r: r)
    cur = (k_shard, v_shard)
    compute_done = None
    for s, j, to, frm in ring_steps(rank, world, direction):
        works, nxt = [], None
        if s + 1 < world:
            nxt = bufs[s % 2]
            with torch.cuda.stream(comm_stream) if cuda else contextlib.nullcontext():
                if compute_done is not None:
                    comm_stream.wait_event(compute_done)  # nxt was read by step s - 1
                ops = [dist.P2POp(dist.isend, cur[0], peer(to), group), dist.P2POp(dist.isend, cur[1], peer(to), group),
                       dist.P2POp(dist.irecv, nxt[0], peer(frm), group),
                       dist.P2POp(dist.irecv, nxt[1], peer(frm), group)]
                works = dist.batch_isend_irecv(ops)
        with torch.cuda.stream(compute_stream) if cuda else contextlib.nullcontext():
            step_fn(s, j, cur[0], cur[1], s == 0, s == world - 1)
            if cuda:
                compute_done = torch.cuda.Event()
                compute_done.record(compute_stream)
            for w in works:
                w.wait()  # CUDA: the compute stream waits for the transfer; CPU: blocks
        if nxt is not None:
            cur = nxt
    if cuda:
        torch.cuda.current_stream(k_shard.device).wait_stream(compute_stream)


def ring_attention_distributed(q_shard, k_shard, v_shard, causal: bool = True, layout: str = "striped",
                               scale: float | None = None, group=None, stream=None, comm_stream=None):
    """Exact attention with the sequence spread over the ranks of `group`, one shard each.

    Rank r of N holds shard r (under `layout`) of an S = N*Sq token sequence:
    q_shard [B,Hq,Sq,D] and k_shard/v_shard [B,Hkv,Sq,D], bf16 (or fp32), CUDA, in
    shard-local order. Returns this rank's (out [B,Hq,Sq,D], lse [B,Hq,Sq]) in
    shard-local order. The KV shards cross between GPUs by NCCL point-to-point into
    this GPU's buffers; the kernel reads only this GPU's memory.
    """
    import torch.distributed as dist

    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    B, Hq, Sq, D = q_shard.shape
    S = world * Sq
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dev = q_shard.device
    o_acc = torch.empty((B, Hq, Sq, D), dtype=torch.float32, device=dev) if world > 1 else None
    lse_acc = torch.empty((B, Hq, Sq), dtype=torch.float32, device=dev) if world > 1 else None
    out = torch.empty_like(q_shard)
    lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=dev)
    compute = stream or torch.cuda.current_stream(dev)

    def step(s, j, kc, vc, first, last):
        ring_attention_ring_step(q_shard, kc, vc, S, world, rank, j, causal, layout, scale, first, last, o_acc,
                                 lse_acc, out, lse, stream=compute)

    run_ring_pass(k_shard, v_shard, step, group, 1, compute, comm_stream)
    return out, lse


def run_backward_ring(k_shard, v_shard, acc_like, step_kv, step_q, group=None, compute_stream=None, comm_stream=None):
    """The transfers of the backward ring for one rank; returns (dK, dV) of the rank's own
    KV shard, in K's dtype.

    At step s the rank holds KV shard j = (rank + s) mod world with its dK/dV accumulators
    (fp32, shaped like `acc_like`). step_kv(s, j, k, v, acc_k, acc_v, fin_k, fin_v, first,
    last) folds the rank's query shard into them (on the last step into fin_k/fin_v, bf16);
    step_q(s, j, k, v, first, last) folds KV shard j into the rank's dQ. K and V move on
    to rank - 1 while step s runs; the accumulators leave once step_kv has run, while
    step_q runs; the next step waits for both. After the last step each rank holds the
    finished dK/dV of shard rank - 1 and sends them home. CUDA tensors use NCCL and
    streams; CPU tensors (gloo) take the same order synchronously.
    """
    import torch.distributed as dist

    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    cuda = k_shard.is_cuda
    if cuda:
        compute_stream = compute_stream or torch.cuda.current_stream(k_shard.device)
        comm_stream = comm_stream or torch.cuda.Stream(k_shard.device)
        comm_stream.wait_stream(compute_stream)
    peer = (lambda r: dist.get_global_rank(group, r)) if group is not None else (lambda r: r)
    to, frm = peer((rank - 1) % world), peer((rank + 1) % world)  # blocks move to rank - 1
    kv_bufs = [(torch.empty_like(k_shard), torch.empty_like(v_shard)) for _ in range(2 if world > 1 else 0)]
    acc_bufs = [(torch.empty_like(acc_like), torch.empty_like(acc_like)) for _ in range(2 if world > 1 else 0)]
    fin_k, fin_v = torch.empty_like(k_shard), torch.empty_like(v_shard)
    cur_kv = (k_shard, v_shard)
    cur_acc = acc_bufs[0] if world > 1 else (None, None)
    on_comm = (lambda: torch.cuda.stream(comm_stream)) if cuda else contextlib.nullcontext
    on_compute = (lambda: torch.cuda.stream(compute_stream)) if cuda else contextlib.nullcontext
    compute_done = None
    for s in range(world):
        j = (rank + s) % world
        first, last = s == 0, s == world - 1
        works, nxt_kv, nxt_acc = [], None, None
        if not last:
            nxt_kv = kv_bufs[s % 2]
            with on_comm():
                if compute_done is not None:
                    comm_stream.wait_event(compute_done)  # nxt_kv was read by step s - 1
                works += dist.batch_isend_irecv([
                    dist.P2POp(dist.isend, cur_kv[0], to, group), dist.P2POp(dist.isend, cur_kv[1], to, group),
                    dist.P2POp(dist.irecv, nxt_kv[0], frm, group), dist.P2POp(dist.irecv, nxt_kv[1], frm, group)])
        with on_compute():
            step_kv(s, j, cur_kv[0], cur_kv[1], cur_acc[0], cur_acc[1], fin_k, fin_v, first, last)
            if cuda:
                kv_done = torch.cuda.Event()
                kv_done.record(compute_stream)
        if not last:
            nxt_acc = acc_bufs[(s + 1) % 2]
            with on_comm():
                if cuda:
                    comm_stream.wait_event(kv_done)  # the accumulators leave once this step's part is in
                works += dist.batch_isend_irecv([
                    dist.P2POp(dist.isend, cur_acc[0], to, group), dist.P2POp(dist.isend, cur_acc[1], to, group),
                    dist.P2POp(dist.irecv, nxt_acc[0], frm, group), dist.P2POp(dist.irecv, nxt_acc[1], frm, group)])
        with on_compute():
            step_q(s, j, cur_kv[0], cur_kv[1], first, last)
            if cuda:
                compute_done = torch.cuda.Event()
                compute_done.record(compute_stream)
            for w in works:
                w.wait()
        if not last:
            cur_kv, cur_acc = nxt_kv, nxt_acc
    if world == 1:
        return fin_k, fin_v
    # the shard finished here is rank - 1's: send it home, receive this rank's own
    home_k, home_v = torch.empty_like(k_shard), torch.empty_like(v_shard)
    with on_comm():
        if cuda:
            comm_stream.wait_stream(compute_stream)
        works = dist.batch_isend_irecv([
            dist.P2POp(dist.isend, fin_k, to, group), dist.P2POp(dist.isend, fin_v, to, group),
            dist.P2POp(dist.irecv, home_k, frm, group), dist.P2POp(dist.irecv, home_v, frm, group)])
    with on_compute():
        for w in works:
            w.wait()
    if cuda:
        torch.cuda.current_stream(k_shard.device).wait_stream(compute_stream)
    return home_k, home_v


def ring_attention_backward_distributed(q_shard, k_shard, v_shard, out_shard, lse_shard, dout_shard,
                                        causal: bool = True, layout: str = "striped", scale: float | None = None,
                                        group=None, stream=None, comm_stream=None):
    """Gradients (dq, dk, dv) of this rank's shards for attention spread over the ranks of
    `group` (the forward of ring_attention_distributed): the backward ring of the
    RingAttention deep-architecture article, section "activation checkpointing and memory
    recomputation". All tensors are this rank's shard in shard-local order; out_shard and
    lse_shard are the forward's results. The per-step arithmetic runs in the library's
    kernels (ring_attn_bwd_ring_step); this function moves the shards."""
    import torch.distributed as dist

    from .api import ring_backward_prep, ring_backward_step

    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    B, Hq, Sq, D = q_shard.shape
    S = world * Sq
    compute = stream or torch.cuda.current_stream(q_shard.device)
    ws = ring_backward_prep(out_shard, lse_shard, dout_shard, S, world, rank, causal, layout, stream=compute)
    dq_acc = torch.empty((B, Hq, Sq, D), dtype=torch.float32, device=q_shard.device) if world > 1 else None
    dq = torch.empty_like(q_shard)
    acc_like = torch.empty(k_shard.shape, dtype=torch.float32, device=q_shard.device)

    def step_kv(s, j, kc, vc, acc_k, acc_v, fin_k, fin_v, first, last):
        ring_backward_step(q_shard, dout_shard, kc, vc, S, world, rank, j, ws, causal, layout, scale, parts=1,
                           first=first, last=last, dk_acc=acc_k, dv_acc=acc_v, dk=fin_k, dv=fin_v, stream=compute)

    def step_q(s, j, kc, vc, first, last):
        ring_backward_step(q_shard, dout_shard, kc, vc, S, world, rank, j, ws, causal, layout, scale, parts=2,
                           first=first, last=last, dq_acc=dq_acc, dq=dq, stream=compute)

    dk, dv = run_backward_ring(k_shard, v_shard, acc_like, step_kv, step_q, group, compute, comm_stream)
    return dq, dk, dv


# ------------------------------------------------------------------ virtual ranks on one device

class PlanOp(NamedTuple):
    """One operation of a virtual ring, in issue order.

    name:   (kind, rank, step) (step -1 for the per-rank operations before and after the
            steps); unique within a plan.
    stream: ("compute", rank) or ("copy", rank). Operations of one stream run in order.
    reads, writes: the buffers it touches (names as in the plan builders).
    waits:  names of earlier operations whose completion it waits for (an event recorded
            right after each one was issued)."""
    name: tuple
    stream: tuple
    reads: tuple
    writes: tuple
    waits: tuple


def forward_ring_plan(P: int) -> list:
    """The operations of VirtualRing.run: P virtual ranks of the forward ring.

    Buffers: ("kv", r) is rank r's own K/V shard, ("buf", r, i) its two receive buffers,
    ("state", r) its running state and output. Step s of rank r ("step") folds the shard
    it holds, (r - s) mod P (RingAttention deep-architecture article, section 2); its copy
    ("copy") pulls rank r - 1's current shard into buffer s % 2, which rank r holds at
    step s + 1. A copy waits for this rank's step s - 1 (which read the buffer), for rank
    r + 1's copy at s - 1 (which read it too) and for rank r - 1's copy at s - 1 (which
    filled the source); a step waits for the copy that filled what it reads."""
    def cur(r, s):
        return ("kv", r) if s == 0 else ("buf", r, (s - 1) % 2)

    ops = []
    for s in range(P):
        for r in range(P):
            waits = (("copy", r, s - 1),) if s > 0 else ()
            reads = (cur(r, s),) if s == 0 else (cur(r, s), ("state", r))
            ops.append(PlanOp(("step", r, s), ("compute", r), reads, (("state", r),), waits))
        if s + 1 < P:
            for r in range(P):
                prev, nxt = (r - 1) % P, (r + 1) % P
                waits = (("step", r, s - 1), ("copy", nxt, s - 1), ("copy", prev, s - 1)) if s > 0 else ()
                ops.append(PlanOp(("copy", r, s), ("copy", r), (cur(prev, s),), (("buf", r, s % 2),), waits))
    return ops


def backward_ring_plan(P: int) -> list:
    """The operations of VirtualBackwardRing.run: P virtual ranks of the backward ring.

    Buffers: ("in", r) rank r's query-side inputs (q, dO, out, lse), ("stats", r) its row
    statistics, ("kv", r) its own K/V shard, ("kvbuf", r, i) two receive buffers,
    ("acc", r, i) two dK/dV accumulator buffers (one when P = 1), ("dq", r) its dQ
    accumulator and output, ("fin", r) the finished dK/dV of the shard it ends with,
    ("home", r) its own dK/dV. At step s rank r holds KV shard (r + s) mod P (the backward
    ring of the RingAttention deep-architecture article, section "activation checkpointing
    and memory recomputation") with its accumulators: "step_kv" folds rank r's query shard
    into them (on the last step into "fin"), "step_q" folds the shard into rank r's dQ.
    Rank r's copies pull rank r + 1's K/V ("copy_kv") and, once rank r + 1's step_kv is
    in, its accumulators ("copy_acc"); "home" pulls rank r's finished gradients from rank
    r + 1 after the last step."""
    def kv(r, s):
        return ("kv", r) if s == 0 else ("kvbuf", r, (s - 1) % 2)

    def acc(r, s):
        return ("acc", r, s % 2) if P > 1 else ("acc", r, 0)

    ops = [PlanOp(("prep", r, -1), ("compute", r), (("in", r),), (("stats", r),), ()) for r in range(P)]
    for s in range(P):
        first, last = s == 0, s == P - 1
        for r in range(P):
            waits = (("copy_kv", r, s - 1), ("copy_acc", r, s - 1)) if s > 0 else ()
            reads = (("in", r), ("stats", r), kv(r, s)) + (() if first else (acc(r, s),))
            ops.append(PlanOp(("step_kv", r, s), ("compute", r), reads, (("fin", r),) if last else (acc(r, s),),
                              waits))
            reads = (("in", r), ("stats", r), kv(r, s)) + (() if first else (("dq", r),))
            ops.append(PlanOp(("step_q", r, s), ("compute", r), reads, (("dq", r),), ()))
        if last:
            break
        for r in range(P):
            src, dst = (r + 1) % P, (r - 1) % P  # blocks move to rank - 1
            waits = (("step_q", r, s - 1), ("copy_kv", dst, s - 1), ("copy_acc", dst, s - 1),
                     ("copy_kv", src, s - 1)) if s > 0 else ()
            ops.append(PlanOp(("copy_kv", r, s), ("copy", r), (kv(src, s),), (("kvbuf", r, s % 2),), waits))
            ops.append(PlanOp(("copy_acc", r, s), ("copy", r), (acc(src, s),), (acc(r, s + 1),),
                              (("step_kv", src, s),)))
    for r in range(P):
        src = (r + 1) % P
        ops.append(PlanOp(("home", r, -1), ("copy", r), (("fin", src),), (("home", r),), (("step_q", src, P - 1),)))
    return ops


def _issue_plan(ops, streams, execute, timing: bool):
    """Issues `ops` in order: each waits for the events of its `waits`, runs execute(op)
    on its stream, then records its event. Returns {name: event}."""
    events = {}
    for op in ops:
        stream = streams[op.stream]
        for w in op.waits:
            stream.wait_event(events[w])
        with torch.cuda.stream(stream):
            execute(op, stream)
        e = torch.cuda.Event(enable_timing=timing)
        e.record(stream)
        events[op.name] = e
    return events


class VirtualRing:
    """P virtual ranks of the forward ring on one device, each with its own query shard,
    KV double buffer, running state, workspace, compute stream and copy stream.

    run() issues forward_ring_plan(P): rank r's step s folds the KV shard it holds into
    its state on its compute stream; meanwhile its copy stream pulls the previous rank's
    current shard into its other buffer (a device-to-device copy). Events order the
    streams as the plan says; no kernel waits on another kernel.
    """

    def __init__(self, q_shards, k_shards, v_shards, causal=True, layout="striped", scale=None):
        self.P = len(q_shards)
        if not (len(k_shards) == len(v_shards) == self.P) or self.P < 1:
            raise ValueError("one q, k and v shard per rank")
        B, Hq, Sq, D = q_shards[0].shape
        self.S = self.P * Sq
        self.causal, self.layout = causal, layout
        self.scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
        self.dev = q_shards[0].device
        self.q, self.k, self.v = list(q_shards), list(k_shards), list(v_shards)
        P = self.P
        self.bufs = [[(torch.empty_like(k_shards[r]), torch.empty_like(v_shards[r])) for _ in range(2)]
                     for r in range(P)] if P > 1 else [[] for _ in range(P)]
        self.o_acc = [torch.empty((B, Hq, Sq, D), dtype=torch.float32, device=self.dev) for _ in range(P)]
        self.lse_acc = [torch.empty((B, Hq, Sq), dtype=torch.float32, device=self.dev) for _ in range(P)]
        self.out = [torch.empty_like(q_shards[r]) for r in range(P)]
        self.lse = [torch.empty((B, Hq, Sq), dtype=torch.float32, device=self.dev) for _ in range(P)]
        from . import binding as _b
        wsb = _b.ring_attn_fwd_workspace_bytes(B, Hq, k_shards[0].shape[1], self.S, D, P, int(causal),
                                               {"contiguous": 0, "striped": 1, "zigzag": 2}[layout],
                                               _b.DTYPE_BF16 if q_shards[0].dtype == torch.bfloat16
                                               else _b.DTYPE_FP32)
        if wsb == 0:
            raise _b.RingAttnError(_b.EINVAL, "ring_attn_fwd_workspace_bytes")
        self.ws = [torch.zeros(wsb, dtype=torch.uint8, device=self.dev) for _ in range(P)]
        self.compute = [torch.cuda.Stream(self.dev) for _ in range(P)]
        self.copy = [torch.cuda.Stream(self.dev) for _ in range(P)]
        self.plan = forward_ring_plan(P)

    def _cur(self, r, s):
        return (self.k[r], self.v[r]) if s == 0 else self.bufs[r][(s - 1) % 2]

    def run(self, timing: bool = False):
        """Issue every step of every rank; the caller's current stream waits for all of it.

        With timing, returns per-step CUDA events {"compute": [[(start, end)] per step]
        per rank, "copy": likewise} for the overlap measurement; else None."""
        P = self.P
        caller = torch.cuda.current_stream(self.dev)
        streams = {("compute", r): self.compute[r] for r in range(P)}
        streams.update({("copy", r): self.copy[r] for r in range(P)})
        for st in streams.values():
            st.wait_stream(caller)
        tm = {"compute": [[] for _ in range(P)], "copy": [[] for _ in range(P)]} if timing else None
        starts = {}

        def execute(op, stream):
            kind, r, s = op.name
            if timing:
                starts[op.name] = torch.cuda.Event(enable_timing=True)
                starts[op.name].record(stream)
            if kind == "step":
                kc, vc = self._cur(r, s)
                ring_attention_ring_step(self.q[r], kc, vc, self.S, P, r, (r - s) % P, self.causal, self.layout,
                                         self.scale, s == 0, s == P - 1, self.o_acc[r], self.lse_acc[r],
                                         self.out[r], self.lse[r], workspace=self.ws[r], stream=stream)
            else:
                src_k, src_v = self._cur((r - 1) % P, s)
                dst_k, dst_v = self.bufs[r][s % 2]
                dst_k.copy_(src_k, non_blocking=True)
                dst_v.copy_(src_v, non_blocking=True)

        events = _issue_plan(self.plan, streams, execute, timing)
        for st in streams.values():
            caller.wait_stream(st)
        if timing:
            for op in self.plan:
                kind, r, _ = op.name
                tm["compute" if kind == "step" else "copy"][r].append((starts[op.name], events[op.name]))
        return tm

    def results(self):
        """Per-rank (out [B,Hq,Sq,D], lse [B,Hq,Sq]) in shard-local order."""
        return list(zip(self.out, self.lse))


class VirtualBackwardRing:
    """P virtual ranks of the backward ring on one device (the transfers of
    run_backward_ring as device-to-device copies between the ranks' buffers).

    run() issues backward_ring_plan(P). Rank r keeps query shard r with its dO, out and
    lse; at step s it holds KV shard j = (r + s) mod P and that shard's dK/dV
    accumulators (fp32), runs the dK/dV part (ring_attn_bwd_ring_step, parts = KV) then
    the dQ part (parts = Q) on its compute stream, and its copy stream pulls rank r + 1's
    K/V and (once rank r + 1's dK/dV part is in) accumulators into its other buffers.
    After the last step each rank holds the finished gradients of shard r - 1 and copies
    them home. Events order the streams; no kernel waits on another.
    """

    def __init__(self, q_shards, k_shards, v_shards, out_shards, lse_shards, dout_shards, causal=True,
                 layout="striped", scale=None):
        self.P = P = len(q_shards)
        if P < 1 or not all(len(x) == P for x in (k_shards, v_shards, out_shards, lse_shards, dout_shards)):
            raise ValueError("one shard of each tensor per rank")
        B, Hq, Sq, D = q_shards[0].shape
        self.S = P * Sq
        self.causal, self.layout = causal, layout
        self.scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
        self.dev = q_shards[0].device
        self.q, self.k, self.v = list(q_shards), list(k_shards), list(v_shards)
        self.out, self.lse, self.dout = list(out_shards), list(lse_shards), list(dout_shards)
        f32 = dict(dtype=torch.float32, device=self.dev)
        two = 2 if P > 1 else 0
        self.kv_bufs = [[(torch.empty_like(k_shards[r]), torch.empty_like(v_shards[r])) for _ in range(two)]
                        for r in range(P)]
        self.acc_bufs = [[(torch.empty(k_shards[r].shape, **f32), torch.empty(v_shards[r].shape, **f32))
                          for _ in range(max(two, 1))] for r in range(P)]
        self.dq_acc = [torch.empty(q_shards[r].shape, **f32) if P > 1 else None for r in range(P)]
        self.dq = [torch.empty_like(q_shards[r]) for r in range(P)]
        self.fin = [(torch.empty_like(k_shards[r]), torch.empty_like(v_shards[r])) for r in range(P)]
        self.dk = [torch.empty_like(k_shards[r]) for r in range(P)]
        self.dv = [torch.empty_like(v_shards[r]) for r in range(P)]
        from . import binding as _b
        wsb = _b.ring_attn_bwd_ring_workspace_bytes(B, Hq, Hq, self.S, D, P, int(causal),
                                                    {"contiguous": 0, "striped": 1, "zigzag": 2}[layout],
                                                    _b.DTYPE_BF16)
        if wsb == 0:
            raise _b.RingAttnError(_b.EINVAL, "ring_attn_bwd_ring_workspace_bytes")
        self.ws = [torch.zeros(wsb, dtype=torch.uint8, device=self.dev) for _ in range(P)]
        self.compute = [torch.cuda.Stream(self.dev) for _ in range(P)]
        self.copy = [torch.cuda.Stream(self.dev) for _ in range(P)]
        self.plan = backward_ring_plan(P)

    def _kv(self, r, s):
        return (self.k[r], self.v[r]) if s == 0 else self.kv_bufs[r][(s - 1) % 2]

    def _acc(self, r, s):
        return self.acc_bufs[r][s % 2] if self.P > 1 else self.acc_bufs[r][0]

    def run(self, timing: bool = False):
        """Issue the plan; the caller's current stream waits for all of it. With timing,
        returns (start, end) CUDA events {"compute": per rank, one per step (both parts),
        "copy": per rank, two per step (K/V, then the accumulators)}; else None."""
        from .api import ring_backward_prep, ring_backward_step

        P = self.P
        caller = torch.cuda.current_stream(self.dev)
        streams = {("compute", r): self.compute[r] for r in range(P)}
        streams.update({("copy", r): self.copy[r] for r in range(P)})
        for st in streams.values():
            st.wait_stream(caller)
        tm = {"compute": [[] for _ in range(P)], "copy": [[] for _ in range(P)]} if timing else None
        starts = {}

        def execute(op, stream):
            kind, r, s = op.name
            if timing:
                starts[op.name] = torch.cuda.Event(enable_timing=True)
                starts[op.name].record(stream)
            first, last = s == 0, s == P - 1
            if kind == "prep":
                ring_backward_prep(self.out[r], self.lse[r], self.dout[r], self.S, P, r, self.causal, self.layout,
                                   workspace=self.ws[r], stream=stream)
            elif kind == "step_kv":
                kc, vc = self._kv(r, s)
                ak, av = self._acc(r, s)
                fk, fv = self.fin[r]
                ring_backward_step(self.q[r], self.dout[r], kc, vc, self.S, P, r, (r + s) % P, self.ws[r],
                                   self.causal, self.layout, self.scale, parts=1, first=first, last=last,
                                   dk_acc=ak, dv_acc=av, dk=fk, dv=fv, stream=stream)
            elif kind == "step_q":
                kc, vc = self._kv(r, s)
                ring_backward_step(self.q[r], self.dout[r], kc, vc, self.S, P, r, (r + s) % P, self.ws[r],
                                   self.causal, self.layout, self.scale, parts=2, first=first, last=last,
                                   dq_acc=self.dq_acc[r], dq=self.dq[r], stream=stream)
            elif kind == "copy_kv":
                dk_, dv_ = self.kv_bufs[r][s % 2]
                sk, sv = self._kv((r + 1) % P, s)
                dk_.copy_(sk, non_blocking=True)
                dv_.copy_(sv, non_blocking=True)
            elif kind == "copy_acc":
                na, nb = self._acc(r, s + 1)
                sa, sb = self._acc((r + 1) % P, s)
                na.copy_(sa, non_blocking=True)
                nb.copy_(sb, non_blocking=True)
            else:  # home
                src = (r + 1) % P
                self.dk[r].copy_(self.fin[src][0], non_blocking=True)
                self.dv[r].copy_(self.fin[src][1], non_blocking=True)

        events = _issue_plan(self.plan, streams, execute, timing)
        for st in streams.values():
            caller.wait_stream(st)
        if timing:
            for op in self.plan:
                kind, r, s = op.name
                if kind == "step_q":
                    tm["compute"][r].append((starts[("step_kv", r, s)], events[op.name]))
                elif kind in ("copy_kv", "copy_acc"):
                    tm["copy"][r].append((starts[op.name], events[op.name]))
        return tm

    def results(self):
        """Per-rank (dq [B,Hq,Sq,D], dk [B,Hkv,Sq,D], dv [B,Hkv,Sq,D]) in shard-local order."""
        return list(zip(self.dq, self.dk, self.dv))
