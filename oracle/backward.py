"""fp64 CPU oracle for the backward pass of exact (ring) attention.

TEST INFRASTRUCTURE ONLY, like the rest of this package: nothing on the product
path may import, call or execute it. It shares no code with the CUDA path.

Sources:
  [RECOMP] RingAttention deep-architecture article (techknowgenie), section
           "activation checkpointing and memory recomputation": for the backward
           pass only the queries and the row statistics (m, l) of the forward are
           kept; K and V blocks travel the ring in the opposite direction and the
           attention map is recomputed in place.
  [DEF]    FlashAttention video summary (aitrends), chapter "basic attention
           computation": O = softmax(scale * Q K^T) V with row max subtraction.

The pages give no gradient formulas. Those used here are the chain rule applied
to [DEF], with the statistics saved as lse = m + ln l (one number per row):
    P  = exp(S - lse)                 S = scale * Q K^T, masked entries give P = 0
    dV = P^T dO                       dP = dO V^T
    Delta_t = sum_u P_tu dP_tu = <dO_t, O_t>
    dS = P * (dP - Delta)             (elementwise, Delta broadcast along keys)
    dQ = scale * dS K                 dK = scale * dS^T Q
Under GQA, dK and dV of a kv head sum the contributions of every query head that
reads it. The tests pin these against central finite differences of [DEF] and
against torch autograd, so the formulas are checked, not assumed.

All arithmetic is fp64 on the exact values of the (already rounded) inputs.
"""
from __future__ import annotations

import numpy as np

from .attention import _as_f64, allowed_keys, block_allowed, kv_head, shard_tokens


def _mask(S: int, causal: bool) -> np.ndarray:
    """[S, S] allowed-pair mask on global token order: key u visible to query t iff u <= t."""
    t = np.arange(S)
    return t[None, :] < allowed_keys(t, S, causal)[:, None] if causal else np.ones((S, S), dtype=bool)


def attention_backward_reference(q, k, v, dout, causal: bool, scale: float):
    """Gradients (dq [B,Hq,S,D], dk, dv [B,Hkv,S,D]) of O = attention(q, k, v) against dout.

    Everything is formed from the plain definition: the full masked score matrix of
    each head, its exact softmax, O and lse, then the formulas in the module header.
    """
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    dq = np.zeros((B, Hq, S, D))
    dk = np.zeros((B, Hkv, S, D))
    dv = np.zeros((B, Hkv, S, D))
    mask = _mask(S, causal)
    for b in range(B):
        for h in range(Hq):
            g = kv_head(h, Hq, Hkv)
            Q, K, V, dO = _as_f64(q[b, h]), _as_f64(k[b, g]), _as_f64(v[b, g]), _as_f64(dout[b, h])
            s = np.where(mask, scale * (Q @ K.T), -np.inf)
            m = s.max(axis=1, keepdims=True)
            p = np.exp(s - m)
            p /= p.sum(axis=1, keepdims=True)
            O = p @ V
            dP = dO @ V.T
            delta = np.sum(dO * O, axis=1, keepdims=True)
            dS = p * (dP - delta)
            dq[b, h] = scale * (dS @ K)
            dk[b, g] += scale * (dS.T @ Q)
            dv[b, g] += p.T @ dO
    return dq, dk, dv


def delta_rows(out, dout) -> np.ndarray:
    """Delta [B,Hq,S] = <dO_t, O_t> for every row (the row sum of P * dP)."""
    return np.sum(_as_f64(out) * _as_f64(dout), axis=-1)


def ring_attention_backward_online(q, k, v, dout, out, lse, P: int, causal: bool, layout: str, scale: float):
    """The backward pass in ring form [RECOMP], in fp64.

    Query shard i keeps Q_i, dO_i, the saved lse_i and Delta_i = <dO_i, O_i>. The KV
    blocks travel the ring in the opposite direction to the forward pass: at step
    s = 0..P-1 query shard i meets KV shard j = (i + s) mod P. Each meeting
    recomputes S = scale Q_i K_j^T on the block's mask and P = exp(S - lse_i), then
    adds dQ_i += scale dS K_j while dK_j += scale dS^T Q_i and dV_j += P^T dO_i ride
    along with the KV block. `out` and `lse` are the forward results.
    """
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    dq = np.zeros((B, Hq, S, D))
    dk = np.zeros((B, Hkv, S, D))
    dv = np.zeros((B, Hkv, S, D))
    shards = [shard_tokens(S, P, layout, i) for i in range(P)]
    L = _as_f64(lse)
    Dl = delta_rows(out, dout)
    for b in range(B):
        for h in range(Hq):
            g = kv_head(h, Hq, Hkv)
            Qa, Ka, Va, dOa = _as_f64(q[b, h]), _as_f64(k[b, g]), _as_f64(v[b, g]), _as_f64(dout[b, h])
            for i in range(P):
                tq = shards[i]
                for s in range(P):
                    j = (i + s) % P
                    tk = shards[j]
                    allowed = block_allowed(tq, tk, causal)
                    Sij = scale * (Qa[tq] @ Ka[tk].T)
                    Pij = np.where(allowed, np.exp(np.where(allowed, Sij, 0.0) - L[b, h, tq][:, None]), 0.0)
                    dPij = dOa[tq] @ Va[tk].T
                    dSij = Pij * (dPij - Dl[b, h, tq][:, None])
                    dq[b, h, tq] += scale * (dSij @ Ka[tk])
                    dk[b, g, tk] += scale * (dSij.T @ Qa[tq])
                    dv[b, g, tk] += Pij.T @ dOa[tq]
    return dq, dk, dv


def backward_rows_dq(q, k, v, dout, rows, causal: bool, scale: float) -> np.ndarray:
    """dQ for selected (b, h, t) rows only: one materialised score row each (O(S D) per row)."""
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    res = np.zeros((len(rows), D))
    for n, (b, h, t) in enumerate(rows):
        g = kv_head(h, Hq, Hkv)
        na = allowed_keys(t, S, causal)
        K, V = _as_f64(k[b, g, :na]), _as_f64(v[b, g, :na])
        qt, dot = _as_f64(q[b, h, t]), _as_f64(dout[b, h, t])
        s = scale * (K @ qt)
        p = np.exp(s - s.max())
        p /= p.sum()
        dP = V @ dot
        delta = float(p @ dP)           # = <dO_t, O_t> with O_t = p V
        res[n] = scale * ((p * (dP - delta)) @ K)
    return res


def backward_rows_dkdv(q, k, v, dout, keys, causal: bool, scale: float):
    """dK and dV for selected (b, g, u) key rows of kv head g.

    Key u collects from every query t it is visible to (all t >= u when causal), over
    the query heads of its GQA group; each such query row's softmax is formed from
    its own materialised score row, so this is cheap only for keys seen by few rows.
    """
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    dk = np.zeros((len(keys), D))
    dv = np.zeros((len(keys), D))
    for n, (b, g, u) in enumerate(keys):
        ts = np.arange(u if causal else 0, S)
        for h in range(Hq):
            if kv_head(h, Hq, Hkv) != g:
                continue
            K, V = _as_f64(k[b, g]), _as_f64(v[b, g])
            Q, dO = _as_f64(q[b, h, ts]), _as_f64(dout[b, h, ts])
            s = scale * (Q @ K.T)                                   # [len(ts), S]
            if causal:
                s = np.where(np.arange(S)[None, :] <= ts[:, None], s, -np.inf)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            dP = dO @ V.T
            delta = np.sum(p * dP, axis=1)
            dS_col = p[:, u] * (dP[:, u] - delta)                   # column u of dS
            dk[n] += scale * (dS_col @ Q)
            dv[n] += p[:, u] @ dO
    return dk, dv
