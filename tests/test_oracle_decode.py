"""Pins for the fp64 decode oracle: closed forms, the full-attention definition, the split."""
import math

import numpy as np
import pytest

import oracle


def rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def test_decode_is_the_last_row_of_noncausal_attention():
    """A decode query is an ordinary query row that sees every key."""
    B, Hq, Hkv, S, D = 2, 4, 2, 37, 8
    k, v = rand((B, Hkv, S, D), 1), rand((B, Hkv, S, D), 2)
    q1 = rand((B, Hq, D), 3)
    q = np.zeros((B, Hq, S, D))
    q[:, :, 5] = q1
    O, L = oracle.attention_rows(q, k, v, [(b, h, 5) for b in range(B) for h in range(Hq)], False, 0.3)
    Od, Ld = oracle.decode_reference(q1, k, v, 0.3)
    np.testing.assert_allclose(Od.reshape(-1, D), O, atol=1e-13)
    np.testing.assert_allclose(Ld.reshape(-1), L, atol=1e-13)


def test_uniform_keys_closed_form():
    """All keys equal: O = mean of V, lse = s + ln S."""
    S, D = 50, 4
    kr = rand((D,), 4)
    k = np.broadcast_to(kr, (1, 1, S, D)).copy()
    v = rand((1, 1, S, D), 5)
    q1 = rand((1, 1, D), 6)
    O, L = oracle.decode_reference(q1, k, v, 0.7)
    np.testing.assert_allclose(O[0, 0], v[0, 0].mean(axis=0), atol=1e-14)
    assert abs(L[0, 0] - (0.7 * float(q1[0, 0] @ kr) + math.log(S))) < 1e-12


def test_dominant_key_returns_its_value():
    S, D = 64, 8
    k = rand((1, 1, S, D), 7) * 0.01
    q1 = np.ones((1, 1, D))
    k[0, 0, 41] = 40.0  # score margin >= 300
    v = rand((1, 1, S, D), 8)
    O, _ = oracle.decode_reference(q1, k, v, 1.0)
    np.testing.assert_allclose(O[0, 0], v[0, 0, 41], atol=1e-12)


@pytest.mark.parametrize("P,layout,chunk", [(1, "contiguous", 7), (4, "striped", 3), (4, "zigzag", 5),
                                            (8, "contiguous", 64)])
def test_split_and_merge_equals_full(P, layout, chunk):
    B, Hq, Hkv, S, D = 1, 4, 1, 64, 6
    k, v = rand((B, Hkv, S, D), 9), rand((B, Hkv, S, D), 10)
    q1 = rand((B, Hq, D), 11)
    O1, L1 = oracle.decode_reference(q1, k, v, 0.5)
    O2, L2 = oracle.decode_split(q1, k, v, P, layout, chunk, 0.5)
    np.testing.assert_allclose(O2, O1, atol=1e-13)
    np.testing.assert_allclose(L2, L1, atol=1e-13)
