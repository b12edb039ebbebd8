"""The virtual rings' operation plans on the host: every ordering the streams and events
allow gives the same result.

VirtualRing and VirtualBackwardRing issue forward_ring_plan / backward_ring_plan: each
operation runs on one stream (operations of a stream run in order) after the events of
the operations it waits for. A GPU parity test can pass by the luck of timing even with a
missing wait, so these tests check the plans themselves:
  * a wait names an operation issued earlier (a CUDA stream waits for the last record of
    an event at the time of the call, so a later record would be no wait at all);
  * no two operations that the streams and events leave unordered touch one buffer
    where either writes it (no race in any interleaving);
  * run in issue order with symbolic buffer contents, every step reads the shard the
    ring schedule names (RingAttention deep-architecture article: section 2 forward,
    (r - s) mod P; section "activation checkpointing and memory recomputation" backward,
    (r + s) mod P), every dK/dV accumulator gathers one part from every rank and ends at
    its home rank, and every dQ / state gathers every KV shard.
A plan with one wait taken out must fail the race check (the check has teeth).
"""
import pytest

from sequence_exact_attention_ring_b200 import ring


def happens_before(ops):
    """For each op (by index), the set of indices of ops ordered before it by its stream
    and by waits, transitively."""
    index = {op.name: i for i, op in enumerate(ops)}
    last_on_stream = {}
    before = []
    for i, op in enumerate(ops):
        preds = set()
        if op.stream in last_on_stream:
            preds.add(last_on_stream[op.stream])
        for w in op.waits:
            assert w in index and index[w] < i, f"{op.name} waits for {w}, not issued before it"
            preds.add(index[w])
        closure = set(preds)
        for p in preds:
            closure |= before[p]
        before.append(closure)
        last_on_stream[op.stream] = i
    return before


def races(ops):
    before = happens_before(ops)
    found = []
    for j, b in enumerate(ops):
        for i in range(j):
            if i in before[j]:
                continue
            a = ops[i]
            wa, wb = set(a.writes), set(b.writes)
            ra, rb = set(a.reads), set(b.reads)
            clash = (wa & (rb | wb)) | (ra & wb)
            if clash:
                found.append((a.name, b.name, sorted(clash)))
    return found


@pytest.mark.parametrize("P", [1, 2, 3, 4, 5, 8])
def test_forward_plan_has_no_race_and_follows_the_ring(P):
    ops = ring.forward_ring_plan(P)
    assert len({op.name for op in ops}) == len(ops)
    assert races(ops) == []
    # symbolic run in issue order
    val = {("kv", r): ("KV", r) for r in range(P)}
    state = {r: [] for r in range(P)}
    for op in ops:
        kind, r, s = op.name
        if kind == "step":
            held = val[op.reads[0]]
            assert held == ("KV", (r - s) % P), (op.name, held)
            state[r].append(held[1])
        else:
            (dst,) = op.writes
            val[dst] = val[op.reads[0]]
    for r in range(P):
        assert state[r] == [(r - s) % P for s in range(P)]


@pytest.mark.parametrize("P", [1, 2, 3, 4, 5, 8])
def test_backward_plan_has_no_race_and_gathers_every_part(P):
    ops = ring.backward_ring_plan(P)
    assert len({op.name for op in ops}) == len(ops)
    assert races(ops) == []
    val = {("kv", r): ("KV", r) for r in range(P)}
    dq = {r: [] for r in range(P)}
    for op in ops:
        kind, r, s = op.name
        if kind == "prep":
            val[("stats", r)] = ("STATS", r)
        elif kind in ("step_kv", "step_q"):
            j = (r + s) % P
            kv_buf = [b for b in op.reads if b[0] in ("kv", "kvbuf")]
            assert len(kv_buf) == 1 and val[kv_buf[0]] == ("KV", j), (op.name, val.get(kv_buf[0]))
            assert val[("stats", r)] == ("STATS", r)
            if kind == "step_q":
                dq[r].append(j)
                continue
            acc_in = [b for b in op.reads if b[0] == "acc"]
            parts = () if s == 0 else val[acc_in[0]][2]
            if s > 0:
                assert val[acc_in[0]][:2] == ("ACC", j)
            new = ("ACC", j, parts + (r,))
            (dst,) = op.writes
            val[dst] = ("FIN", j, new[2]) if s == P - 1 else new
        else:  # copies and home
            (dst,) = op.writes
            val[dst] = val[op.reads[0]]
    for r in range(P):
        assert sorted(dq[r]) == list(range(P))
        fin = val[("home", r)]
        assert fin[:2] == ("FIN", r) and sorted(fin[2]) == list(range(P)), fin


def test_a_missing_wait_is_caught():
    """Each wait of the plans guards something: taking out any single one of them (for
    P = 4) leaves a race, except waits implied by another path through the streams."""
    for build in (ring.forward_ring_plan, ring.backward_ring_plan):
        ops = build(4)
        caught = 0
        removable = 0
        for i, op in enumerate(ops):
            for w in op.waits:
                cut = list(ops)
                cut[i] = op._replace(waits=tuple(x for x in op.waits if x != w))
                if races(cut):
                    caught += 1
                else:
                    removable += 1
        assert caught > 0
        # the copy of the source's readiness (a wait on the neighbour's previous copy) and
        # the accumulators' readiness are each necessary
        op = next(o for o in ops if o.name[0] in ("copy", "copy_kv") and o.name[2] == 1)
        w = ("copy", (op.name[1] - 1) % 4, 0) if op.name[0] == "copy" else ("copy_kv", (op.name[1] + 1) % 4, 0)
        cut = [o._replace(waits=tuple(x for x in o.waits if x != w)) if o is op else o for o in ops]
        assert races(cut), f"{build.__name__}: removing {w} from {op.name} left no race"


def test_backward_plan_accumulator_copy_needs_the_step():
    ops = ring.backward_ring_plan(3)
    cut = [o._replace(waits=()) if o.name[0] == "copy_acc" else o for o in ops]
    assert any(a[0] == "step_kv" and b[0] == "copy_acc" for a, b, _ in races(cut))
