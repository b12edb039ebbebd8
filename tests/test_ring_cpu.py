"""The ring across ranks on the host: schedule, shard maps and the send/receive/swap
bookkeeping of run_ring_pass with world-size 2 and 3 gloo ranks.

No attention is computed here: the step function records which KV shard each rank
holds at each step (the shards carry their index as their values), so the test checks
the transfers and the order, forward and backward ring.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from sequence_exact_attention_ring_b200 import ring

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_ring_steps_forward_and_backward():
    # RingAttention deep-architecture article, section 2: rank r holds shard (r - s) mod N
    for world in (1, 2, 5):
        for r in range(world):
            fwd = ring.ring_steps(r, world, 1)
            bwd = ring.ring_steps(r, world, -1)
            assert [x[1] for x in fwd] == [(r - s) % world for s in range(world)]
            assert [x[1] for x in bwd] == [(r + s) % world for s in range(world)]
            assert all(x[2] == (r + 1) % world and x[3] == (r - 1) % world for x in fwd)
            assert all(x[2] == (r - 1) % world and x[3] == (r + 1) % world for x in bwd)
            # every shard is visited once, own shard first
            assert sorted(x[1] for x in fwd) == list(range(world)) and fwd[0][1] == r
    with pytest.raises(ValueError):
        ring.ring_steps(0, 2, 0)


@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
def test_shard_token_index_matches_the_oracle_map(layout):
    """Two independent statements of the shard map agree (oracle.shard_tokens is the
    oracle's own; shard_token_index prepares ring inputs)."""
    S, P = 48, 4
    for i in range(P):
        np.testing.assert_array_equal(ring.shard_token_index(S, P, layout, i).numpy(),
                                      oracle.shard_tokens(S, P, layout, i))


@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
def test_split_and_join_shards_round_trip(layout):
    x = torch.arange(2 * 3 * 24 * 5, dtype=torch.float32).view(2, 3, 24, 5)
    sh = ring.split_shards(x, 4, layout)
    assert len(sh) == 4 and all(s.shape == (2, 3, 6, 5) and s.is_contiguous() for s in sh)
    assert torch.equal(ring.join_shards(sh, layout), x)
    toks = ring.shard_token_index(24, 4, layout, 2)
    assert torch.equal(sh[2], x[:, :, toks])


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, direction, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist
    from sequence_exact_attention_ring_b200 import ring as rg
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # this rank's K/V shard carries its index (K) and 100 + index (V)
        k = torch.full((1, 2, 3, 4), float(rank))
        v = torch.full((1, 2, 3, 4), float(100 + rank))
        seen = []

        def step(s, j, kc, vc, first, last):
            seen.append((s, j, float(kc.unique().item()), float(vc.unique().item()), first, last,
                         kc.data_ptr() == k.data_ptr()))

        rg.run_ring_pass(k, v, step, direction=direction)
        q.put((rank, seen, float(k.unique().item()), float(v.unique().item())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("direction", [1, -1])
def test_ring_pass_bookkeeping_with_gloo_ranks(world, direction):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, direction, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, seen, k0, v0 in res:
        assert [x[0] for x in seen] == list(range(world))
        for s, j, kv, vv, first, last, own in seen:
            assert j == (rank - direction * s) % world        # the shard the schedule names
            assert kv == j and vv == 100 + j                  # is the shard that arrived
            assert first == (s == 0) and last == (s == world - 1)
            assert own == (s == 0)                            # step 0 uses the rank's own buffers
        assert (k0, v0) == (rank, 100 + rank)                 # the caller's shard is never overwritten


def _bwd_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist
    from sequence_exact_attention_ring_b200 import ring as rg
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # the rank's KV shard carries its index; each rank adds rank + 1 to dK and 10 (rank + 1) to dV
        k = torch.full((1, 2, 3, 4), float(rank))
        v = torch.full((1, 2, 3, 4), float(100 + rank))
        acc_like = torch.empty((1, 2, 3, 4))
        seen = []

        def step_kv(s, j, kc, vc, acc_k, acc_v, fin_k, fin_v, first, last):
            assert float(kc.unique().item()) == j and float(vc.unique().item()) == 100 + j
            prev_k = 0.0 if first else acc_k.clone()
            prev_v = 0.0 if first else acc_v.clone()
            if last:  # finished: tag with the shard index so the test sees where it ends up
                fin_k.copy_(prev_k + (rank + 1) + 1000 * j)
                fin_v.copy_(prev_v + 10 * (rank + 1) + 1000 * j)
            else:
                acc_k.copy_(prev_k + (rank + 1))
                acc_v.copy_(prev_v + 10 * (rank + 1))
            seen.append(("kv", s, j, first, last))

        def step_q(s, j, kc, vc, first, last):
            seen.append(("q", s, j, first, last))

        dk, dv = rg.run_backward_ring(k, v, acc_like, step_kv, step_q)
        q.put((rank, seen, float(dk.unique().item()), float(dv.unique().item())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_backward_ring_accumulators_collect_every_rank_and_return_home(world):
    """The backward ring (RingAttention deep-architecture article, section "activation
    checkpointing and memory recomputation"): rank r holds KV shard (r + s) mod world at step s,
    the dK/dV accumulators travel with it and gather one part from every rank, and the
    finished gradients of shard r end at rank r."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bwd_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    total = world * (world + 1) // 2
    for rank, seen, dk, dv in res:
        kv = [x for x in seen if x[0] == "kv"]
        qq = [x for x in seen if x[0] == "q"]
        assert [x[2] for x in kv] == [(rank + s) % world for s in range(world)]
        assert [x[2] for x in qq] == [(rank + s) % world for s in range(world)]
        assert all(x[3] == (x[1] == 0) and x[4] == (x[1] == world - 1) for x in seen)
        assert dk == total + 1000 * rank and dv == 10 * total + 1000 * rank
