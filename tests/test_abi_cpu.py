"""The C-ABI library on the host: symbols, argument errors, the exact schedule.

No compute call is made here (no GPU in this environment); every check runs on
host code paths that return before touching CUDA.
"""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import oracle
from sequence_exact_attention_ring_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ringattn.h")


@pytest.fixture(scope="module")
def lib():
    from sequence_exact_attention_ring_b200 import build
    build.build()
    return B.load()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ring_attn_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = header_functions()
    assert len(names) >= 10
    nm = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (ring_attn_\w+)", nm))
    for n in names:
        assert n in exported, n
        assert hasattr(lib, n)
        assert n in B.SIGNATURES, f"binding lacks {n}"


def test_version_and_strerror(lib):
    assert B.ring_attn_version() >= 100
    for code in (B.OK, B.EINVAL, B.EALIGN, B.EUNSUPPORTED, B.EWORKSPACE, B.ECUDA, B.ETIMEOUT):
        assert B.strerror(code) != "unknown error"
    assert B.strerror(-99) == "unknown error"


GOOD = dict(B=1, Hq=4, Hkv=2, S=1024, D=128, P=4, causal=1, layout=1, dtype=1)
FAKE = 0x10000  # aligned, never dereferenced: every call below fails validation first


def fwd(scale=0.1, **kw):
    a = dict(GOOD)
    ptrs = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, ws=FAKE, wsb=256)
    for key in list(kw):
        if key in ptrs:
            ptrs[key] = kw.pop(key)
    a.update(kw)
    return B.ring_attn_fwd(ptrs["q"], ptrs["k"], ptrs["v"], ptrs["out"], ptrs["lse"], a["B"], a["Hq"], a["Hkv"],
                           a["S"], a["D"], a["P"], a["causal"], a["layout"], scale, a["dtype"], ptrs["ws"],
                           ptrs["wsb"], None)


@pytest.mark.parametrize("bad,code", [
    (dict(B=0), B.EINVAL), (dict(Hq=0), B.EINVAL), (dict(S=0), B.EINVAL), (dict(P=0), B.EINVAL),
    (dict(S=1000, P=3), B.EINVAL), (dict(Hq=3, Hkv=2), B.EINVAL), (dict(causal=2), B.EINVAL),
    (dict(layout=5), B.EINVAL), (dict(layout=2, S=1020), B.EINVAL), (dict(dtype=7), B.EINVAL),
    (dict(D=96), B.EUNSUPPORTED),
    (dict(D=256), B.EUNSUPPORTED), (dict(q=0), B.EINVAL), (dict(lse=0), B.EINVAL),
    (dict(k=FAKE + 8), B.EALIGN), (dict(out=FAKE + 2), B.EALIGN), (dict(ws=0), B.EWORKSPACE),
    (dict(wsb=16), B.EWORKSPACE), (dict(scale=0.0), B.EINVAL), (dict(scale=-1.0), B.EINVAL),
    (dict(scale=float("inf")), B.EINVAL), (dict(scale=float("nan")), B.EINVAL),
])
def test_fwd_rejects_bad_arguments(lib, bad, code):
    assert fwd(**bad) == code


def test_workspace_bytes(lib):
    assert B.ring_attn_fwd_workspace_bytes(1, 8, 8, 16384, 128, 8, 1, 0, 1) >= 256
    assert B.ring_attn_fwd_workspace_bytes(1, 8, 8, 16383, 128, 8, 1, 0, 1) == 0
    assert B.ring_attn_fwd_workspace_bytes(1, 8, 3, 16384, 128, 8, 1, 0, 1) == 0


def test_step_and_merge_reject_bad_arguments(lib):
    assert B.ring_attn_fwd_step(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 2, 64, 64, 4, 4, 0, 1, 1, 0.1, 1, 0, FAKE, 256,
                                None) == B.EINVAL
    assert B.ring_attn_fwd_step(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 2, 64, 64, 4, 0, -1, 1, 1, 0.1, 1, 0, FAKE,
                                256, None) == B.EINVAL
    assert B.ring_attn_merge(FAKE, FAKE, 0, 10, 128, FAKE, FAKE, 1, None) == B.EINVAL
    assert B.ring_attn_merge(FAKE, FAKE, 2, 10, 12, FAKE, FAKE, 1, None) == B.EINVAL
    assert B.ring_attn_merge(FAKE, FAKE, 2, 10, 128, FAKE, FAKE, 3, None) == B.EINVAL
    assert B.ring_attn_merge(FAKE + 4, FAKE, 2, 10, 128, FAKE, FAKE, 1, None) == B.EALIGN
    assert B.ring_attn_debug_watchdog(0, FAKE, 256, None) == B.EINVAL
    assert B.ring_attn_debug_watchdog(100, FAKE, 8, None) == B.EWORKSPACE


# ------------------------------------------------------------------ schedule

def visit_counts(S, P, causal, layout, tq, tk):
    counts = np.zeros((S, S), dtype=np.int32)
    n = B.ring_attn_debug_visit_counts(S, P, causal, layout, tq, tk, counts.ctypes.data)
    assert n >= 0
    return counts, n


@pytest.mark.parametrize("S,P", [(8, 1), (8, 2), (24, 3), (24, 8), (64, 4), (96, 8), (256, 8), (512, 16)])
@pytest.mark.parametrize("layout", [0, 1, 2])
@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("tiles", [(4, 4), (8, 2), (6, 5), (256, 128), (64, 32)])
def test_schedule_visits_every_allowed_pair_exactly_once(lib, S, P, layout, causal, tiles):
    if layout == 2 and S % (2 * P):
        assert B.ring_attn_debug_visit_counts(S, P, causal, layout, *tiles, np.zeros(1, np.int32).ctypes.data) < 0
        return
    counts, _ = visit_counts(S, P, causal, layout, *tiles)
    t = np.arange(S)[:, None]
    u = np.arange(S)[None, :]
    # the plain rule on global token order (the oracle's causal rule)
    allowed = u < oracle.allowed_keys(t, S, bool(causal)) if causal else np.ones((S, S), dtype=bool)
    np.testing.assert_array_equal(counts, allowed.astype(np.int32))


def unit_table(Bz, Hq, Hkv, S, P, causal, layout, tq=256):
    nmax = Bz * Hq * P * ((S // P + tq - 1) // tq)
    buf = np.zeros((nmax, 5), dtype=np.int32)
    n = B.ring_attn_debug_decode_units(Bz, Hq, Hkv, S, P, causal, layout, tq, buf.ctypes.data, nmax)
    assert n == nmax
    return buf


@pytest.mark.parametrize("cfg", [(1, 8, 8, 16384, 8, 1, 0), (1, 8, 8, 16384, 8, 1, 1), (2, 32, 8, 131072, 16, 1, 1),
                                 (1, 2, 2, 1024, 4, 0, 0), (1, 4, 1, 4096, 4, 1, 0), (1, 8, 8, 1 << 20, 32, 1, 1),
                                 (1, 8, 8, 16384, 8, 1, 2), (2, 8, 2, 65536, 16, 1, 2), (1, 8, 8, 1 << 20, 32, 1, 2)])
def test_units_cover_each_block_once_in_launch_order(lib, cfg):
    Bz, Hq, Hkv, S, P, causal, layout = cfg
    tab = unit_table(Bz, Hq, Hkv, S, P, causal, layout)
    keys = {tuple(r[:4]) for r in tab}
    nblk = (S // P + 255) // 256
    assert len(keys) == len(tab) == Bz * Hq * P * nblk
    cost = tab[:, 4]
    # the hook describes the D = 64 geometry: the grouped order starts at S * D >= 2^23
    grouped = S * 64 >= 1 << 23
    if not (causal and layout == 2 and grouped):
        # contiguous causal, striped causal, non-causal: longest first over the whole grid
        assert (np.diff(cost) <= 0).all(), "units must be launched longest first"
        if layout == 1 or not causal:
            # block-major: tb descending, inside a tb by (b, kv head, query shard, head)
            order = [(-x[3], x[0], x[1] // (Hq // Hkv), x[2], x[1] % (Hq // Hkv)) for x in tab]
            assert order == sorted(order)
    else:
        # long zigzag causal sequences: consecutive groups of nblk * (Hq/Hkv) units share
        # (b, kv head, query shard), blocks longest first
        rep = Hq // Hkv
        per = nblk * rep
        groups = set()
        for r in range(0, len(tab), per):
            grp = tab[r:r + per]
            key = {(x[0], x[1] // rep, x[2]) for x in grp}
            assert len(key) == 1
            groups |= key
            assert (np.diff(grp[:, 4]) <= 0).all(), "blocks of a group must run longest first"
            assert sorted(grp[:, 3].tolist()) == sorted(list(range(nblk)) * rep)
        assert len(groups) == Bz * Hkv * P


def test_gqa_group_members_are_adjacent_in_launch_order(lib):
    tab = unit_table(2, 32, 8, 131072, 16, 1, 1)
    # consecutive runs of 4 units share (b, kv head, shard, block) and cover the 4 query heads of the group
    for r in range(0, 256, 4):
        grp = tab[r:r + 4]
        assert len({(x[0], x[1] // 4, x[2], x[3]) for x in grp}) == 1
        assert sorted(x[1] % 4 for x in grp) == [0, 1, 2, 3]


@pytest.mark.parametrize("layout", [0, 1, 2])
@pytest.mark.parametrize("causal", [0, 1])
def test_unit_walk_follows_ring_order(lib, layout, causal):
    S, P = 4096, 8
    names = {0: "contiguous", 1: "striped", 2: "zigzag"}
    tab = unit_table(1, 1, 1, S, P, causal, layout)
    for u in range(len(tab)):
        i = tab[u, 2]
        # the unit's last row sees the most keys; shards it cannot see at all are skipped
        a_hi = min(tab[u, 3] * 256 + 255, S // P - 1)
        t_hi = oracle.shard_tokens(S, P, names[layout], i)[a_hi]
        pairs = np.zeros((4096, 2), dtype=np.int32)
        n = B.ring_attn_debug_unit_walk(1, 1, 1, S, P, causal, layout, 256, 128, u, pairs.ctypes.data, 4096)
        assert n == tab[u, 4]
        shards = pairs[:n, 0]
        # ring step s meets kv shard (i - s) mod P: visiting order of distinct shards
        order = [shards[0]] + [s for a, s in zip(shards[:-1], shards[1:]) if s != a]
        expect = [(i - s) % P for s in range(P)]
        if causal:
            expect = [j for j in expect if oracle.shard_tokens(S, P, names[layout], j).min() <= t_hi]
        assert order == expect
        assert order[0] == i
        # inside one shard the key tiles run 0, 1, 2, ...
        for j in set(order):
            kbs = pairs[:n][shards == j, 1]
            np.testing.assert_array_equal(kbs, np.arange(len(kbs)))


@pytest.mark.parametrize("layout,causal", [(1, 1), (1, 0), (0, 0), (2, 0)])
def test_long_block_major_walks_share_one_ring_anchor(lib, layout, causal):
    """Long striped or non-causal launches (S*D >= 2^23): every unit counts the ring from the
    last shard (step s holds shard (P-1-s) mod P), so units of one block index read the same
    shard at the same time; the tiles are the same as on the unit's own ring."""
    S, P = 131072, 8
    names = {0: "contiguous", 1: "striped", 2: "zigzag"}
    tab = unit_table(1, 2, 1, S, P, causal, layout)
    for u in sorted({0, 1, 5, 17, len(tab) // 2, len(tab) - 1}):
        i, tb = int(tab[u, 2]), int(tab[u, 3])
        a_hi = min(tb * 256 + 255, S // P - 1)
        t_hi = int(oracle.shard_tokens(S, P, names[layout], i)[a_hi])
        expect = []
        for s_ in range(P):
            j = (P - 1 - s_) % P
            toks = oracle.shard_tokens(S, P, names[layout], j)
            n_keys = int(np.sum(toks <= t_hi)) if causal else S // P
            expect += [(j, kb) for kb in range((n_keys + 127) // 128)]
        pairs = np.zeros((len(expect) + 8, 2), dtype=np.int32)
        n = B.ring_attn_debug_unit_walk(1, 2, 1, S, P, causal, layout, 256, 128, u, pairs.ctypes.data, len(pairs))
        assert n == len(expect) == tab[u, 4]
        assert [tuple(x) for x in pairs[:n].tolist()] == expect


def test_schedule_info_matches_closed_form_for_1m_striped(lib):
    info = np.zeros(6, dtype=np.int64)
    assert B.ring_attn_debug_schedule_info(1, 8, 8, 1 << 20, 128, 32, 1, 1, info.ctypes.data) == 0
    units, total, partial, longest, first, last = info
    nblk = 32768 // 256
    assert units == 8 * 32 * nblk
    # block tb (256 rows) visits key tiles 0..2tb+1 of each of the 32 shards
    assert total == 8 * 32 * sum(32 * (2 * tb + 2) for tb in range(nblk))
    assert longest == first == 32 * 256 and last == 32 * 2
    # partial tiles: the last two of every shard step of every unit
    assert partial == 8 * 32 * nblk * 32 * 2


# ------------------------------------------------------------------ backward schedule

@pytest.mark.parametrize("S,P,layout", [(256, 1, 0), (256, 2, 1), (768, 3, 0), (1024, 4, 1), (1024, 8, 0),
                                        (1000, 8, 1), (2048, 4, 2), (1536, 3, 2), (3072, 3, 2)])
@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("pass_", [0, 1])
def test_backward_schedule_visits_every_allowed_pair_exactly_once(lib, S, P, layout, causal, pass_):
    """dK/dV pass (KV tiles meeting query tiles) and dQ pass (backward-ring walk)."""
    counts = np.zeros((S, S), dtype=np.int32)
    n = B.ring_attn_debug_bwd_visit_counts(S, P, causal, layout, pass_, counts.ctypes.data)
    assert n > 0
    t = np.arange(S)[:, None]
    u = np.arange(S)[None, :]
    allowed = (u <= t) if causal else np.ones((S, S), dtype=bool)
    np.testing.assert_array_equal(counts, allowed.astype(np.int32))


def test_backward_workspace_and_argument_errors(lib):
    # status header + two fp32 arrays of B*Hq*P*ceil(Sq/128)*128
    assert B.ring_attn_bwd_workspace_bytes(1, 8, 8, 16384, 128, 8, 1, 1, 1) == 256 + 2 * 4 * 8 * 8 * 2048
    assert B.ring_attn_bwd_workspace_bytes(1, 2, 2, 1000, 128, 8, 1, 1, 1) == 256 + 2 * 4 * 2 * 8 * 128
    assert B.ring_attn_bwd_workspace_bytes(1, 8, 8, 16383, 128, 8, 1, 0, 1) == 0
    args = [FAKE] * 9 + [1, 2, 2, 1024, 128, 4, 1, 1, 0.1, 1, FAKE, 1 << 20, None]
    bad = list(args)
    bad[12] = 1022  # S % P != 0
    assert B.ring_attn_bwd(*bad) == B.EINVAL
    bad = list(args)
    bad[5] = 0  # dout null
    assert B.ring_attn_bwd(*bad) == B.EINVAL
    bad = list(args)
    bad[6] = FAKE + 4  # dq misaligned
    assert B.ring_attn_bwd(*bad) == B.EALIGN
    bad = list(args)
    bad[20] = 64  # workspace too small
    assert B.ring_attn_bwd(*bad) == B.EWORKSPACE
    bad = list(args)
    bad[17] = -0.5  # scale
    assert B.ring_attn_bwd(*bad) == B.EINVAL
    bad = list(args)
    bad[13] = 96  # head dim outside {64, 128}
    assert B.ring_attn_bwd(*bad) == B.EUNSUPPORTED


def _code_without_comments(path):
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.sub(r"//[^\n]*", "", text)


def test_noalloc_entry_point_calls_no_allocator():
    """ring_attn_fwd_noalloc and the forward path it calls name no device allocator:
    the no-allocation file and the forward launch code (C ABI, tensor maps, kernels)."""
    csrc = os.path.join(ROOT, "sequence_exact_attention_ring_b200", "csrc")
    files = ["noalloc.cu", "api.cu", "tensor_maps.cu", "fwd_sm100_2sm.cu", "fwd_sm100.cu", "fwd_simt.cu"]
    banned = re.compile(r"\b(cudaMalloc\w*|cudaFree\w*|cuMemAlloc\w*|cuMemFree\w*|cudaMallocAsync|malloc|new\s)")
    for f in files:
        hits = banned.findall(_code_without_comments(os.path.join(csrc, f)))
        assert not hits, f"{f} names {hits}"


def test_noalloc_rejects_bad_arguments_with_the_forward_codes(lib):
    """Argument errors come back before any CUDA call, with ring_attn_fwd's own code."""
    vp = ctypes.c_void_p()
    base = [FAKE] * 5 + [1, 4, 2, 1024, 128, 4, 1, 1, 0.1, 1]
    for idx, val, code in ((8, 1022, B.EINVAL), (9, 96, B.EUNSUPPORTED), (5, 0, B.EINVAL), (12, 7, B.EINVAL)):
        a = list(base)
        a[idx] = val
        assert lib.ring_attn_fwd_noalloc(*a, None, ctypes.byref(vp)) == code, (idx, val)


def test_ring_step_rejects_bad_arguments(lib):
    """ring_attn_fwd_ring_step argument errors come back before any CUDA call."""
    ws = FAKE

    def call(o_acc=FAKE, lse_acc=FAKE, out=FAKE, lse_out=FAKE, q=FAKE, i=0, j=1, flags=0, P=4, S=1024, wsb=256,
             scale=0.1, layout=1):
        return lib.ring_attn_fwd_ring_step(q, FAKE, FAKE, o_acc, lse_acc, out, lse_out, 1, 4, 2, S, 128, P, i, j, 1,
                                           layout, ctypes.c_float(scale), 1, flags, ws, wsb, None)
    assert call(flags=4) == B.EINVAL                      # unknown flag
    assert call(o_acc=None) == B.EINVAL                   # a middle step needs the state
    assert call(lse_acc=None, flags=B.STEP_FIRST) == B.EINVAL
    assert call(out=None, flags=B.STEP_LAST) == B.EINVAL  # a last step needs its outputs
    assert call(q=None) == B.EINVAL
    assert call(i=4) == B.EINVAL and call(j=-1) == B.EINVAL
    assert call(S=1022) == B.EINVAL                       # S % P != 0
    assert call(o_acc=FAKE + 4) == B.EALIGN
    assert call(out=FAKE + 2, flags=B.STEP_LAST) == B.EALIGN
    assert call(wsb=8) == B.EWORKSPACE
    assert call(scale=-1.0) == B.EINVAL
    assert call(layout=3) == B.EINVAL


def test_backward_ring_entry_points_reject_bad_arguments(lib):
    """ring_attn_bwd_ring_prep / _step argument errors come back before any CUDA call."""
    wsb = lib.ring_attn_bwd_ring_workspace_bytes(1, 4, 2, 1024, 128, 4, 1, 1, 1)
    assert wsb == 256 + 2 * 4 * 4 * 256  # header + two statistics of B*Hq*ceil(Sq/128)*128 rows
    assert lib.ring_attn_bwd_ring_workspace_bytes(1, 4, 2, 1022, 128, 4, 1, 1, 1) == 0

    def step(parts=3, flags=0, i=0, j=1, acc=FAKE, out=FAKE, q=FAKE, ws=FAKE, n=wsb, scale=0.1):
        return lib.ring_attn_bwd_ring_step(q, FAKE, FAKE, FAKE, acc, acc, acc, out, out, out, 1, 4, 2, 1024, 128, 4,
                                           i, j, 1, 1, ctypes.c_float(scale), 1, parts, flags, ws, n, None)
    assert step(parts=0) == B.EINVAL and step(parts=4) == B.EINVAL
    assert step(flags=4) == B.EINVAL
    assert step(acc=None) == B.EINVAL                      # a middle step needs the accumulators
    assert step(out=None, flags=B.STEP_LAST) == B.EINVAL   # a last step needs the outputs
    assert step(q=None) == B.EINVAL
    assert step(i=4) == B.EINVAL and step(j=-1) == B.EINVAL
    assert step(acc=FAKE + 8) == B.EALIGN
    assert step(n=wsb - 16) == B.EWORKSPACE
    assert step(scale=0.0) == B.EINVAL
    prep = lib.ring_attn_bwd_ring_prep
    assert prep(FAKE, FAKE, FAKE, 1, 4, 2, 1024, 128, 4, 4, 1, 1, 1, FAKE, wsb, None) == B.EINVAL  # q_index
    assert prep(None, FAKE, FAKE, 1, 4, 2, 1024, 128, 4, 0, 1, 1, 1, FAKE, wsb, None) == B.EINVAL
    assert prep(FAKE, FAKE, FAKE, 1, 4, 2, 1024, 128, 4, 0, 1, 1, 1, FAKE, 64, None) == B.EWORKSPACE
