"""Pins for the fp64 backward oracle.

The oracle's gradient formulas are not on the pages, so they are pinned here to
things that do not depend on them: central finite differences of the plain
forward definition, torch autograd of an independently written forward, closed
forms of special cases, and invariants of softmax. Planted mistakes at the end
show that a slip in a formula fails a pin.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as ob


def rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def case(B=1, Hq=2, Hkv=1, S=7, D=3, seed=0):
    return (rand((B, Hq, S, D), seed), rand((B, Hkv, S, D), seed + 1), rand((B, Hkv, S, D), seed + 2),
            rand((B, Hq, S, D), seed + 3))


def loss(q, k, v, dout, causal, scale):
    """L = sum(O * dO): its gradient with respect to O is dO."""
    O, _ = oracle.attention_reference(q, k, v, causal, scale)
    return float(np.sum(O * dout))


def finite_difference(q, k, v, dout, causal, scale, eps=1e-5):
    grads = []
    for which in range(3):
        arrs = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(arrs[which])
        for idx in np.ndindex(*arrs[which].shape):
            plus = [a.copy() for a in arrs]
            minus = [a.copy() for a in arrs]
            plus[which][idx] += eps
            minus[which][idx] -= eps
            g[idx] = (loss(*plus, dout, causal, scale) - loss(*minus, dout, causal, scale)) / (2 * eps)
        grads.append(g)
    return grads


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Hq,Hkv", [(1, 1), (2, 1), (4, 2)])
def test_gradients_match_central_differences(causal, Hq, Hkv):
    q, k, v, dout = case(1, Hq, Hkv, 6, 3, seed=11 + Hq)
    got = oracle.attention_backward_reference(q, k, v, dout, causal, 0.7)
    ref = finite_difference(q, k, v, dout, causal, 0.7)
    for name, a, b in zip("qkv", got, ref):
        np.testing.assert_allclose(a, b, atol=2e-8, rtol=0, err_msg=f"d{name}")


def test_gradients_match_torch_autograd():
    """An independent forward in torch (fp64), differentiated by autograd."""
    q, k, v, dout = case(2, 4, 2, 12, 5, seed=21)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    kk = tk.repeat_interleave(2, dim=1)
    vv = tv.repeat_interleave(2, dim=1)
    s = 0.45 * tq @ kk.transpose(-1, -2)
    s = s.masked_fill(~torch.ones(12, 12, dtype=torch.bool).tril(), float("-inf"))
    O = torch.softmax(s, dim=-1) @ vv
    (O * torch.tensor(dout)).sum().backward()
    got = oracle.attention_backward_reference(q, k, v, dout, True, 0.45)
    for a, b in zip(got, (tq.grad, tk.grad, tv.grad)):
        np.testing.assert_allclose(a, b.numpy(), atol=1e-12, rtol=0)


def test_single_key_closed_form():
    """One visible key: P = 1, so dV = dO, and dS = dP - <dO, O> = 0 gives dQ = dK = 0."""
    q, k, v, dout = case(1, 1, 1, 1, 4, seed=31)
    dq, dk, dv = oracle.attention_backward_reference(q, k, v, dout, True, 1.0)
    np.testing.assert_allclose(dv, dout, atol=1e-15)
    assert np.abs(dq).max() < 1e-15 and np.abs(dk).max() < 1e-15
    # the causal first row of any sequence sees only key 0: its dQ is zero
    q, k, v, dout = case(1, 1, 1, 9, 4, seed=32)
    dq, _, _ = oracle.attention_backward_reference(q, k, v, dout, True, 1.0)
    assert np.abs(dq[0, 0, 0]).max() < 1e-15


def test_equal_keys_give_zero_dq():
    """All key rows equal: dQ_t = scale * k * sum_u dS_tu = 0 because each dS row sums to 0."""
    q, _, v, dout = case(1, 2, 2, 8, 4, seed=41)
    k = np.broadcast_to(rand((1, 2, 1, 4), 42), (1, 2, 8, 4)).copy()
    dq, _, _ = oracle.attention_backward_reference(q, k, v, dout, True, 0.9)
    assert np.abs(dq).max() < 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_column_sums(causal):
    """sum_u dV_u = sum_t dO_t (rows of P sum to 1) and sum_u dK_u = 0 (rows of dS sum to 0)."""
    q, k, v, dout = case(2, 3, 3, 10, 4, seed=51)
    _, dk, dv = oracle.attention_backward_reference(q, k, v, dout, causal, 0.6)
    np.testing.assert_allclose(dv.sum(axis=2), dout.sum(axis=2), atol=1e-12)
    assert np.abs(dk.sum(axis=2)).max() < 1e-12


@pytest.mark.parametrize("P", [1, 2, 4])
@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_backward_equals_plain(P, layout, causal):
    """The reverse-ring recurrence with the saved lse gives the plain gradients."""
    q, k, v, dout = case(1, 4, 2, 16, 5, seed=61 + P)
    O, L = oracle.attention_reference(q, k, v, causal, 0.4)
    ring = oracle.ring_attention_backward_online(q, k, v, dout, O, L, P, causal, layout, 0.4)
    plain = oracle.attention_backward_reference(q, k, v, dout, causal, 0.4)
    for a, b in zip(ring, plain):
        np.testing.assert_allclose(a, b, atol=1e-12, rtol=0)


@pytest.mark.parametrize("causal", [False, True])
def test_row_blocks_do_not_change_the_gradients(causal):
    """Rows are independent: evaluating them in blocks of 3 or all at once agrees."""
    q, k, v, dout = case(2, 4, 2, 23, 5, seed=67)
    a = oracle.attention_backward_reference(q, k, v, dout, causal, 0.6, row_block=3)
    b = oracle.attention_backward_reference(q, k, v, dout, causal, 0.6, row_block=1024)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, atol=1e-13, rtol=0)


def test_row_and_key_helpers_match_full():
    q, k, v, dout = case(1, 4, 2, 20, 6, seed=71)
    dq, dk, dv = oracle.attention_backward_reference(q, k, v, dout, True, 0.5)
    rows = [(0, 0, 0), (0, 3, 19), (0, 2, 7)]
    np.testing.assert_allclose(oracle.backward_rows_dq(q, k, v, dout, rows, True, 0.5),
                               np.stack([dq[r] for r in rows]), atol=1e-13)
    keys = [(0, 0, 0), (0, 1, 19), (0, 1, 4)]
    gk, gv = oracle.backward_rows_dkdv(q, k, v, dout, keys, True, 0.5)
    np.testing.assert_allclose(gk, np.stack([dk[x] for x in keys]), atol=1e-13)
    np.testing.assert_allclose(gv, np.stack([dv[x] for x in keys]), atol=1e-13)


# ---------------------------------------------------------------- planted mistakes

def _pins_pass():
    try:
        test_gradients_match_central_differences(True, 2, 1)
        test_column_sums(True)
        test_equal_keys_give_zero_dq()
    except AssertionError:
        return False
    return True


def test_pins_pass_on_the_real_oracle():
    assert _pins_pass()


@pytest.mark.parametrize("mistake", ["no_delta", "dk_without_scale", "gqa_last_head_only", "dv_from_ds"])
def test_planted_mistakes_fail_a_pin(monkeypatch, mistake):
    def bad(q, k, v, dout, causal, scale):
        B, Hq, S, D = q.shape
        Hkv = k.shape[1]
        dq = np.zeros((B, Hq, S, D))
        dk = np.zeros((B, Hkv, S, D))
        dv = np.zeros((B, Hkv, S, D))
        mask = np.tril(np.ones((S, S), dtype=bool)) if causal else np.ones((S, S), dtype=bool)
        for b in range(B):
            for h in range(Hq):
                g = h // (Hq // Hkv)
                Q, K, V, dO = q[b, h], k[b, g], v[b, g], dout[b, h]
                s = np.where(mask, scale * (Q @ K.T), -np.inf)
                p = np.exp(s - s.max(axis=1, keepdims=True))
                p /= p.sum(axis=1, keepdims=True)
                dP = dO @ V.T
                delta = 0.0 if mistake == "no_delta" else np.sum(dO * (p @ V), axis=1, keepdims=True)
                dS = p * (dP - delta)
                dq[b, h] = scale * (dS @ K)
                contrib_k = (1.0 if mistake == "dk_without_scale" else scale) * (dS.T @ Q)
                contrib_v = (dS.T @ dO) if mistake == "dv_from_ds" else p.T @ dO
                if mistake == "gqa_last_head_only":
                    dk[b, g] = contrib_k
                    dv[b, g] = contrib_v
                else:
                    dk[b, g] += contrib_k
                    dv[b, g] += contrib_v
        return dq, dk, dv
    monkeypatch.setattr(oracle, "attention_backward_reference", bad)
    assert not _pins_pass(), mistake
