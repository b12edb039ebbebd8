"""fp64 CPU oracle for long-context decode against a sharded KV cache.

TEST INFRASTRUCTURE ONLY, like the rest of this package.

Sources:
  [KV]   RingAttention newsletter (cmlonder), section "code and integration map": in
         production the pain point of inference is the KV cache of a million-token
         prompt; prefill is possible with the ring, and each new token then attends
         to that whole cache.
  [DEF]  FlashAttention video summary (aitrends), chapter "basic attention
         computation": softmax of scaled scores with the row maximum subtracted.
  [EQ]   RingAttention deep-architecture article (techknowgenie), section 3: partial
         results over disjoint key blocks combine by the online-softmax rescale.

A decode step has one new query row per head, at a position after every cached
key, so it sees all S keys (no mask). Its result is the plain definition [DEF] over
the whole cache; a split of the cache into ring shards and chunks, each giving a
normalised partial, merges back to it [EQ].
"""
from __future__ import annotations

import numpy as np

from .attention import _as_f64, kv_head, merge_partials, shard_tokens, softmax_row


def decode_reference(q1, k, v, scale: float):
    """q1 [B,Hq,D] (one query row per head), k/v [B,Hkv,S,D] -> (O [B,Hq,D], lse [B,Hq]) in fp64."""
    B, Hq, D = q1.shape
    Hkv = k.shape[1]
    O = np.zeros((B, Hq, D))
    L = np.zeros((B, Hq))
    for b in range(B):
        for h in range(Hq):
            g = kv_head(h, Hq, Hkv)
            K, V = _as_f64(k[b, g]), _as_f64(v[b, g])
            s = scale * (K @ _as_f64(q1[b, h]))
            p, L[b, h] = softmax_row(s)
            O[b, h] = p @ V
    return O, L


def decode_split(q1, k, v, P: int, layout: str, chunk: int, scale: float):
    """The same step the split way: the cache in P ring shards (layout), each shard in
    chunks of `chunk` local keys; every chunk gives a normalised partial over its keys,
    and the partials merge with the rescale of [EQ]."""
    B, Hq, D = q1.shape
    Hkv, S = k.shape[1], k.shape[2]
    o_parts, l_parts = [], []
    for j in range(P):
        toks = shard_tokens(S, P, layout, j)
        for c0 in range(0, toks.size, chunk):
            sel = toks[c0:c0 + chunk]
            O = np.zeros((B, Hq, D))
            L = np.zeros((B, Hq))
            for b in range(B):
                for h in range(Hq):
                    g = kv_head(h, Hq, Hkv)
                    K, V = _as_f64(k[b, g])[sel], _as_f64(v[b, g])[sel]
                    p, L[b, h] = softmax_row(scale * (K @ _as_f64(q1[b, h])))
                    O[b, h] = p @ V
            o_parts.append(O)
            l_parts.append(L)
    return merge_partials(o_parts, l_parts)
