"""Pins for the fp64 oracle against what the pages and the mathematics fix.

None of these compares the oracle with itself: each expected value is a closed
form, an invariant of softmax attention, a hand-derived case, or a brute-force
evaluation at 60 significant digits. The planted-mistake tests at the end show
that a plausible slip in any one oracle piece fails at least one pin.
"""
import json
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as oa

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def qkv(B=1, Hq=2, Hkv=2, S=16, D=8, seed=0):
    return rand((B, Hq, S, D), seed), rand((B, Hkv, S, D), seed + 1), rand((B, Hkv, S, D), seed + 2)


# ---------------------------------------------------------------- golden fixtures

def test_golden_closed_form_cases():
    cases = json.load(open(os.path.join(GOLDEN, "closed_form_cases.json")))["cases"]
    for c in cases:
        q = np.array(c["q"])[None]
        k = np.array(c["k"])[None]
        v = np.array(c["v"])[None]
        O, L = oracle.attention_reference(q, k, v, c["causal"], c["scale"])
        np.testing.assert_allclose(O[0], np.array(c["expect_o"]), rtol=0, atol=1e-13, err_msg=c["name"])
        np.testing.assert_allclose(L[0], np.array(c["expect_lse"]), rtol=0, atol=1e-13, err_msg=c["name"])
        S = q.shape[2]
        rows = [(0, 0, t) for t in range(S)]
        O2, L2 = oracle.attention_rows(q, k, v, rows, c["causal"], c["scale"])
        np.testing.assert_allclose(O2, np.array(c["expect_o"])[0], atol=1e-13)
        np.testing.assert_allclose(L2, np.array(c["expect_lse"])[0], atol=1e-13)


def test_page_figures_metric_arithmetic():
    """The throughput metric's FLOP count equals the pages' per-step 4*B^2*d summed over blocks."""
    import synthetic
    fig = json.load(open(os.path.join(GOLDEN, "page_figures.json")))
    N = fig["score_matrix_1m"]["N"]
    assert N * N == fig["score_matrix_1m"]["elements"]
    assert 2 * N * N == fig["score_matrix_1m"]["fp16_bytes"]
    # dense: P^2 block steps of 4*Bk^2*d each == 4*S^2*d per head
    for P, S, d in [(4, 1024, 64), (8, 16384, 128), (32, 1048576, 128)]:
        Bk = S // P
        per_step = 4 * Bk * Bk * d
        w = synthetic.custom("x", "bf16", 1, 1, 1, S, d, P, False, "striped", 0)
        assert w.causal_flops() == P * P * per_step
        # the pages' per-step comm bytes (K and V, fp16): 2*2*B*d
        assert 2 * 2 * Bk * d == 2 * (Bk * d * 2)


# ---------------------------------------------------------------- closed forms

@pytest.mark.parametrize("causal", [False, True])
def test_uniform_keys_give_mean_of_allowed_values(causal):
    B, Hq, Hkv, S, D = 1, 4, 2, 24, 8
    q, _, v = qkv(B, Hq, Hkv, S, D, seed=3)
    k = np.broadcast_to(rand((1, Hkv, 1, D), 9), (B, Hkv, S, D)).copy()
    scale = 0.37
    O, L = oracle.attention_reference(q, k, v, causal, scale)
    for h in range(Hq):
        g = h // (Hq // Hkv)
        for t in range(S):
            n = t + 1 if causal else S
            np.testing.assert_allclose(O[0, h, t], v[0, g, :n].mean(axis=0), atol=1e-13)
            s = scale * q[0, h, t] @ k[0, g, 0]
            assert abs(L[0, h, t] - (s + math.log(n))) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_single_dominant_key_returns_its_value(causal):
    """One key beats all others by >= 60 in the scaled logit: O = its V row, lse = its logit.

    Logits are O(1000), so a softmax without max subtraction overflows exp.
    """
    S, D = 16, 4
    q = np.zeros((1, 1, S, D)); q[..., 0] = 1.0
    k = rand((1, 1, S, D), 5) * 0.1 + np.array([1000.0, 0, 0, 0])
    win = 2
    k[0, 0, win, 0] = 1100.0
    v = rand((1, 1, S, D), 6)
    O, L = oracle.attention_reference(q, k, v, causal, scale=1.0)
    for t in range(S):
        if causal and t < win:
            continue
        np.testing.assert_allclose(O[0, 0, t], v[0, 0, win], atol=1e-20 + 1e-30)
        assert abs(L[0, 0, t] - 1.0 * q[0, 0, t] @ k[0, 0, win]) < 1e-9


def test_causal_first_row_is_first_value():
    q, k, v = qkv(2, 4, 1, 32, 16, seed=11)
    scale = 0.25
    O, L = oracle.attention_reference(q, k, v, True, scale)
    for b in range(2):
        for h in range(4):
            np.testing.assert_array_equal(O[b, h, 0], v[b, 0, 0])
            assert L[b, h, 0] == pytest.approx(scale * q[b, h, 0] @ k[b, 0, 0], abs=1e-14)


def test_shift_of_all_keys_shifts_lse_only():
    q, k, v = qkv(1, 2, 2, 20, 8, seed=21)
    w = rand((8,), 99)
    scale = 0.3
    for causal in (False, True):
        O1, L1 = oracle.attention_reference(q, k, v, causal, scale)
        O2, L2 = oracle.attention_reference(q, k + w, v, causal, scale)
        np.testing.assert_allclose(O2, O1, atol=1e-12)
        np.testing.assert_allclose(L2 - L1, scale * q @ w, atol=1e-12)


def test_noncausal_key_permutation_invariance():
    q, k, v = qkv(1, 2, 2, 20, 8, seed=31)
    perm = np.random.default_rng(1).permutation(20)
    O1, L1 = oracle.attention_reference(q, k, v, False, 0.5)
    O2, L2 = oracle.attention_reference(q, k[:, :, perm], v[:, :, perm], False, 0.5)
    np.testing.assert_allclose(O2, O1, atol=1e-12)
    np.testing.assert_allclose(L2, L1, atol=1e-12)


def test_gqa_equals_mha_with_repeated_kv():
    B, Hq, Hkv, S, D = 2, 8, 2, 16, 8
    q, k, v = qkv(B, Hq, Hkv, S, D, seed=41)
    rep = Hq // Hkv
    k_rep = np.repeat(k, rep, axis=1)
    v_rep = np.repeat(v, rep, axis=1)
    for causal in (False, True):
        O1, L1 = oracle.attention_reference(q, k, v, causal, 0.4)
        O2, L2 = oracle.attention_reference(q, k_rep, v_rep, causal, 0.4)
        np.testing.assert_array_equal(O1, O2)
        np.testing.assert_array_equal(L1, L2)


def test_bruteforce_tiny_high_precision():
    """Every row of tiny cases against a 60-digit Decimal evaluation of the definition."""
    getcontext().prec = 60
    for seed, (S, D, causal) in enumerate([(1, 1, False), (3, 2, True), (5, 3, False), (8, 4, True)]):
        q, k, v = qkv(1, 1, 1, S, D, seed=100 + seed)
        scale = 0.7
        O, L = oracle.attention_reference(q, k, v, causal, scale)
        for t in range(S):
            n = t + 1 if causal else S
            s = [Decimal(scale) * sum(Decimal(q[0, 0, t, d]) * Decimal(k[0, 0, u, d]) for d in range(D))
                 for u in range(n)]
            e = [x.exp() for x in s]
            tot = sum(e)
            for d in range(D):
                o = sum(e[u] * Decimal(v[0, 0, u, d]) for u in range(n)) / tot
                assert abs(float(o) - O[0, 0, t, d]) < 1e-14
            assert abs(float(tot.ln()) - L[0, 0, t]) < 1e-14


def test_rows_and_full_agree():
    q, k, v = qkv(2, 4, 2, 40, 8, seed=51)
    rows = [(b, h, t) for b in range(2) for h in range(4) for t in (0, 1, 17, 39)]
    for causal in (False, True):
        O, L = oracle.attention_reference(q, k, v, causal, 0.2)
        O2, L2 = oracle.attention_rows(q, k, v, rows, causal, 0.2)
        for n, (b, h, t) in enumerate(rows):
            np.testing.assert_allclose(O2[n], O[b, h, t], atol=1e-13)
            assert abs(L2[n] - L[b, h, t]) < 1e-13


# ---------------------------------------------------------------- the ring recurrence

def test_shard_maps():
    np.testing.assert_array_equal(oracle.shard_tokens(12, 3, "contiguous", 1), [4, 5, 6, 7])
    np.testing.assert_array_equal(oracle.shard_tokens(12, 3, "striped", 1), [1, 4, 7, 10])
    # zigzag: 2P chunks of S/(2P) tokens, shard i holds chunks i and 2P-1-i
    np.testing.assert_array_equal(oracle.shard_tokens(16, 2, "zigzag", 0), [0, 1, 2, 3, 12, 13, 14, 15])
    np.testing.assert_array_equal(oracle.shard_tokens(16, 2, "zigzag", 1), [4, 5, 6, 7, 8, 9, 10, 11])
    for layout in ("contiguous", "striped", "zigzag"):
        allt = np.concatenate([oracle.shard_tokens(24, 4, layout, i) for i in range(4)])
        np.testing.assert_array_equal(np.sort(allt), np.arange(24))
    with pytest.raises(ValueError):
        oracle.shard_tokens(10, 3, "striped", 0)
    with pytest.raises(ValueError):
        oracle.shard_tokens(12, 4, "zigzag", 0)  # S % 2P != 0


def _causal_pairs_per_shard(S, P, layout):
    """(query, key) pairs each query shard folds under the causal mask, over all ring steps."""
    counts = []
    for i in range(P):
        tq = oracle.shard_tokens(S, P, layout, i)
        counts.append(sum(int(oracle.block_allowed(tq, oracle.shard_tokens(S, P, layout, j), True).sum())
                          for j in range(P)))
    return counts


@pytest.mark.parametrize("S,P", [(16, 2), (48, 4), (64, 8)])
def test_causal_work_per_shard_closed_forms(S, P):
    """Contiguous: shard i folds i full blocks and one triangle, i*Sq^2 + Sq(Sq+1)/2 pairs.
    Zigzag: chunks i and 2P-1-i together see 2P-1 full chunks and two triangles,
    (2P-1)C^2 + C(C+1) pairs for every shard, so the ring is balanced."""
    Sq, C = S // P, S // (2 * P)
    assert _causal_pairs_per_shard(S, P, "contiguous") == [i * Sq * Sq + Sq * (Sq + 1) // 2 for i in range(P)]
    assert _causal_pairs_per_shard(S, P, "zigzag") == [(2 * P - 1) * C * C + C * (C + 1)] * P
    assert sum(_causal_pairs_per_shard(S, P, "striped")) == S * (S + 1) // 2


@pytest.mark.parametrize("P", [1, 2, 4, 8])
@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
@pytest.mark.parametrize("causal", [False, True])
def test_online_ring_equals_full_softmax(P, layout, causal):
    q, k, v = qkv(1, 4, 2, 32, 8, seed=61 + P)
    O1, L1 = oracle.attention_reference(q, k, v, causal, 0.35)
    O2, L2 = oracle.ring_attention_online(q, k, v, P, causal, layout, 0.35)
    np.testing.assert_allclose(O2, O1, atol=1e-12, rtol=0)
    np.testing.assert_allclose(L2, L1, atol=1e-12, rtol=0)


def test_online_ring_heavy_logits_no_nan():
    q, k, v = qkv(1, 2, 2, 32, 8, seed=71)
    k = k * 30.0
    for layout in ("contiguous", "striped", "zigzag"):
        O1, L1 = oracle.attention_reference(q, k, v, True, 1.0)
        O2, L2 = oracle.ring_attention_online(q, k, v, 8, True, layout, 1.0)
        assert np.isfinite(O2).all() and np.isfinite(L2).all()
        np.testing.assert_allclose(O2, O1, atol=1e-10)
        np.testing.assert_allclose(L2, L1, rtol=1e-13, atol=1e-10)


def _lazy_speculative_ring(q, k, v, P, causal, layout, scale, tile, cap=2.0 ** 20, thresh=8.0):
    """The tensor-core kernels' block rule, restated in fp64 (a check of the rule, not
    the oracle): base-2 exponentials against a reference maximum m that moves lazily. A
    block is first exponentiated against the current m and kept when its row sum stays
    <= cap; otherwise (and for a row's first visible block) the block maximum is taken, and
    m moves to it when it exceeds m by more than thresh, rescaling l and O."""
    B, Hq, S, D = q.shape
    rep = Hq // k.shape[1]
    c = scale / math.log(2.0)
    O = np.zeros(q.shape)
    L = np.full(q.shape[:3], -np.inf)
    with np.errstate(over="ignore", invalid="ignore"):
        for b in range(B):
            for h in range(Hq):
                g = h // rep
                for i in range(P):
                    tq = oracle.shard_tokens(S, P, layout, i)
                    m = np.full(len(tq), -np.inf)
                    l = np.zeros(len(tq))
                    o = np.zeros((len(tq), D))
                    for s in range(P):
                        tk = oracle.shard_tokens(S, P, layout, (i - s) % P)
                        for kb in range(0, len(tk), tile):
                            tkb = tk[kb:kb + tile]
                            x = (q[b, h, tq] @ k[b, g, tkb].T) * c
                            x[~oracle.block_allowed(tq, tkb, causal)] = -np.inf
                            p = np.exp2(x - np.where(np.isfinite(m), m, 0.0)[:, None])
                            keep = np.isfinite(m) & (p.sum(1) <= cap)
                            mb = x.max(1)
                            move = ~keep & (mb > m + thresh)
                            alpha = np.where(np.isfinite(m), np.exp2(m - mb), 0.0)
                            l = np.where(move, l * alpha, l)
                            o = np.where(move[:, None], o * alpha[:, None], o)
                            m = np.where(move, mb, m)
                            redo = np.exp2(x - np.where(np.isfinite(m), m, 0.0)[:, None])
                            p = np.where(keep[:, None], p, redo)
                            l = l + p.sum(1)
                            o = o + p @ v[b, g, tkb]
                    O[b, h, tq] = o / l[:, None]
                    L[b, h, tq] = (m + np.log2(l)) * math.log(2.0)
    return O, L


@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
@pytest.mark.parametrize("pattern", ["plain", "rising", "jump"])
@pytest.mark.parametrize("cap", [2.0 ** 20, 1.0])
def test_lazy_speculative_reference_maximum_equals_full_softmax(layout, pattern, cap):
    """O/l and lse do not depend on the reference maximum the exponentials use, as long as
    nothing overflows: the kernels' speculative block rule equals full softmax (cap = 1
    forces the exact-maximum path on almost every block)."""
    q, k, v = qkv(1, 2, 2, 64, 8, seed=91)
    if pattern == "rising":
        k = k * (1.0 + 6.0 * np.arange(64) / 64.0)[None, None, :, None]
    elif pattern == "jump":
        k[:, :, [5, 23, 40]] *= 400.0
    O1, L1 = oracle.attention_reference(q, k, v, True, 0.5)
    O2, L2 = _lazy_speculative_ring(q, k, v, 4, True, layout, 0.5, tile=4, cap=cap)
    assert np.isfinite(O2).all() and np.isfinite(L2).all()
    np.testing.assert_allclose(O2, O1, atol=1e-11, rtol=0)
    np.testing.assert_allclose(L2, L1, rtol=1e-12, atol=1e-11)


def test_speculative_rule_needs_a_finite_cap():
    """Accepting every speculative block (no cap) lets a score far above the reference
    overflow: the sum check is what keeps the rule exact."""
    q, k, v = qkv(1, 2, 2, 64, 8, seed=91)
    k[:, :, [5, 23, 40]] *= 400.0
    O2, L2 = _lazy_speculative_ring(q, k, v, 4, True, "striped", 0.5, tile=4, cap=np.inf)
    assert not (np.isfinite(O2).all() and np.isfinite(L2).all())


# ---------------------------------------------------------------- merge

def _partition_partials(q, k, v, causal, scale, labels, n_parts):
    B, Hq, S, D = q.shape
    base = np.ones((B, Hq, S, S), dtype=bool)
    if causal:
        base &= np.tril(np.ones((S, S), dtype=bool))[None, None]
    parts = []
    for p in range(n_parts):
        mask = base & (labels == p)[None, None, None, :]
        parts.append(oracle.attention_keyset(q, k, v, mask, scale))
    return parts


@pytest.mark.parametrize("causal", [False, True])
def test_merge_of_any_key_partition_equals_full(causal):
    q, k, v = qkv(1, 2, 2, 24, 8, seed=81)
    labels = np.random.default_rng(3).integers(0, 4, size=24)
    parts = _partition_partials(q, k, v, causal, 0.5, labels, 4)
    O, L = oracle.merge_partials([p[0] for p in parts], [p[1] for p in parts])
    Of, Lf = oracle.attention_reference(q, k, v, causal, 0.5)
    np.testing.assert_allclose(O, Of, atol=1e-12)
    np.testing.assert_allclose(L, Lf, atol=1e-12)
    # order independence
    rev = parts[::-1]
    O2, L2 = oracle.merge_partials([p[0] for p in rev], [p[1] for p in rev])
    np.testing.assert_allclose(O2, O, atol=1e-14)
    np.testing.assert_allclose(L2, L, atol=1e-14)


def test_merge_empty_part_is_identity_and_all_empty_is_zero():
    rows, D = 5, 4
    o = rand((rows, D), 1)
    lse = rand((rows,), 2)
    empty_o = rand((rows, D), 3)                  # garbage values must be ignored
    empty_l = np.full(rows, -np.inf)
    O, L = oracle.merge_partials([o, empty_o], [lse, empty_l])
    np.testing.assert_allclose(O, o, atol=0)
    np.testing.assert_allclose(L, lse, atol=0)
    O, L = oracle.merge_partials([empty_o, empty_o], [empty_l, empty_l])
    assert (O == 0).all() and np.isneginf(L).all()


def test_merge_two_parts_closed_form():
    """lse1 = ln 1, lse2 = ln 3: weights 1/4 and 3/4, merged lse = ln 4."""
    o1 = np.array([[4.0, 0.0]])
    o2 = np.array([[0.0, 8.0]])
    O, L = oracle.merge_partials([o1, o2], [np.array([0.0]), np.array([math.log(3.0)])])
    np.testing.assert_allclose(O, [[1.0, 6.0]], atol=1e-15)
    assert abs(L[0] - math.log(4.0)) < 1e-15


# ---------------------------------------------------------------- planted mistakes

def _pins_pass():
    try:
        test_golden_closed_form_cases()
        test_causal_first_row_is_first_value()
        test_uniform_keys_give_mean_of_allowed_values(True)
        test_single_dominant_key_returns_its_value(False)
        test_gqa_equals_mha_with_repeated_kv()
        for layout in ("contiguous", "striped", "zigzag"):
            test_online_ring_equals_full_softmax(4, layout, True)
        test_shard_maps()
        test_causal_work_per_shard_closed_forms(48, 4)
        test_merge_two_parts_closed_form()
    except (AssertionError, FloatingPointError, ValueError, IndexError):
        return False
    return True


def test_pins_pass_on_the_real_oracle():
    assert _pins_pass()


@pytest.mark.parametrize("mistake", ["exclusive_diagonal", "no_max_subtraction", "wrong_gqa_map",
                                     "striped_transposed", "zigzag_shifted_pairing", "merge_no_weight"])
def test_planted_mistakes_fail_a_pin(monkeypatch, mistake):
    if mistake == "exclusive_diagonal":
        monkeypatch.setattr(oa, "allowed_keys",
                            lambda t, S, causal: (t if causal else (S if np.isscalar(t) else np.full_like(t, S))))
    elif mistake == "no_max_subtraction":
        def bad(s):
            p = np.exp(s)
            return p, np.zeros(s.shape[:-1] + (1,)), np.sum(p, axis=-1, keepdims=True)
        monkeypatch.setattr(oa, "softmax_stats", bad)
    elif mistake == "wrong_gqa_map":
        monkeypatch.setattr(oa, "kv_head", lambda h, Hq, Hkv: h % Hkv)
    elif mistake == "striped_transposed":
        real = oa.shard_tokens

        def bad(S, P, layout, i):
            t = real(S, P, layout, i)
            # local index and shard index swapped: i*P + a instead of a*P + i
            return (i * P + np.arange(S // P)) if layout == "striped" else t
        monkeypatch.setattr(oa, "shard_tokens", bad)
    elif mistake == "zigzag_shifted_pairing":
        real = oa.shard_tokens

        def bad(S, P, layout, i):
            if layout != "zigzag":
                return real(S, P, layout, i)
            # pairs chunk i with chunk P+i: still a partition, but not the balanced one
            C = S // (2 * P)
            c = np.arange(C)
            return np.concatenate([i * C + c, (P + i) * C + c])
        monkeypatch.setattr(oa, "shard_tokens", bad)
        monkeypatch.setattr(oracle, "shard_tokens", bad)
    elif mistake == "merge_no_weight":
        def bad(o_parts, lse_parts):
            return np.mean(np.stack(o_parts), axis=0), np.log(np.sum(np.exp(np.stack(lse_parts)), axis=0))
        monkeypatch.setattr(oa, "merge_partials", bad)
        monkeypatch.setattr(oracle, "merge_partials", bad)
    with np.errstate(all="ignore"):
        assert not _pins_pass(), f"planted mistake {mistake} went unnoticed"
