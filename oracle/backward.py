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


def attention_backward_reference(q, k, v, dout, causal: bool, scale: float, row_block: int = 1024):
    """Gradients (dq [B,Hq,S,D], dk, dv [B,Hkv,S,D]) of O = attention(q, k, v) against dout.

    Everything is formed from the plain definition, the formulas in the module header,
    one block of query rows at a time (rows are independent; a block only bounds the
    memory of the materialised score rows): the block's masked score rows (keys u <= t
    when causal), their exact softmax, O and Delta, then dS. dq of the block follows
    from its own rows; dk and dv sum the contributions of every row, block by block.
    """
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    dq = np.zeros((B, Hq, S, D))
    dk = np.zeros((B, Hkv, S, D))
    dv = np.zeros((B, Hkv, S, D))
    for b in range(B):
        for g in range(Hkv):
            K, V = _as_f64(k[b, g]), _as_f64(v[b, g])
            for h in range(Hq):
                if kv_head(h, Hq, Hkv) != g:
                    continue
                Q, dO = _as_f64(q[b, h]), _as_f64(dout[b, h])
                for r0 in range(0, S, row_block):
                    r1 = min(S, r0 + row_block)
                    kmax = r1 if causal else S      # no row of the block sees a key at or past r1
                    s = Q[r0:r1] @ K[:kmax].T
                    s *= scale
                    if causal:
                        # keys u > t inside the block's own token range are masked
                        # (every key below r0 is visible to every row of the block)
                        t = np.arange(r0, r1)
                        diag = s[:, r0:r1]
                        diag[np.arange(r0, r1)[None, :] >= allowed_keys(t, S, causal)[:, None]] = -np.inf
                    p = s                               # exp(s - m) / l, in place
                    p -= p.max(axis=1, keepdims=True)
                    np.exp(p, out=p)
                    p /= p.sum(axis=1, keepdims=True)
                    O = p @ V[:kmax]
                    dS = dO[r0:r1] @ V[:kmax].T         # dP, then dS = P * (dP - Delta) in place
                    dS -= np.sum(dO[r0:r1] * O, axis=1, keepdims=True)
                    dS *= p
                    dq[b, h, r0:r1] = scale * (dS @ K[:kmax])
                    dk[b, g, :kmax] += scale * (dS.T @ Q[r0:r1])
                    dv[b, g, :kmax] += p.T @ dO[r0:r1]
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


def backward_rows_dq(q, k, v, dout, rows, causal: bool, scale: float, chunk: int = 64) -> np.ndarray:
    """dQ for selected (b, h, t) rows only: one materialised score row each (O(S D) per row).

    Rows of one head are evaluated together (one matrix product for their score rows);
    each row keeps its own allowed keys, softmax and Delta.
    """
    rows = list(rows)
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    res = np.zeros((len(rows), D))
    by_head: dict[tuple[int, int], list[int]] = {}
    for n, (b, h, t) in enumerate(rows):
        by_head.setdefault((b, h), []).append(n)
    kv_cache: dict[tuple[int, int], tuple[np.ndarray, np.ndarray]] = {}
    for (b, h), idxs in sorted(by_head.items()):
        g = kv_head(h, Hq, Hkv)
        if (b, g) not in kv_cache:
            kv_cache.clear()
            kv_cache[(b, g)] = (_as_f64(k[b, g]), _as_f64(v[b, g]))
        K, V = kv_cache[(b, g)]
        for c0 in range(0, len(idxs), chunk):
            part = idxs[c0:c0 + chunk]
            ts = [rows[n][2] for n in part]
            qs, dos = _as_f64(q[b, h][ts]), _as_f64(dout[b, h][ts])
            kmax = max(allowed_keys(t, S, causal) for t in ts)
            s_all = scale * (qs @ K[:kmax].T)                      # [n, kmax]
            dP_all = dos @ V[:kmax].T
            for r, (n, t) in enumerate(zip(part, ts)):
                na = allowed_keys(t, S, causal)
                s = s_all[r, :na]
                p = np.exp(s - s.max())
                p /= p.sum()
                dP = dP_all[r, :na]
                delta = float(p @ dP)           # = <dO_t, O_t> with O_t = p V
                res[n] = scale * ((p * (dP - delta)) @ K[:na])
    return res


def backward_rows_dkdv(q, k, v, dout, keys, causal: bool, scale: float, row_block: int = 1024):
    """dK and dV for selected (b, g, u) key rows of kv head g.

    Key u collects from every query t it is visible to (all t >= u when causal), over
    the query heads of its GQA group; each such query row's softmax is formed from
    its own materialised score row (rows in blocks of row_block), so this is cheap
    only for keys seen by few rows.
    """
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    keys = list(keys)
    dk = np.zeros((len(keys), D))
    dv = np.zeros((len(keys), D))
    by_group: dict[tuple[int, int], list[int]] = {}
    for n, (b, g, u) in enumerate(keys):
        by_group.setdefault((b, g), []).append(n)
    for (b, g), idxs in sorted(by_group.items()):
        us = np.array([keys[n][2] for n in idxs])
        K, V = _as_f64(k[b, g]), _as_f64(v[b, g])
        t0 = int(us.min()) if causal else 0
        for h in range(Hq):
            if kv_head(h, Hq, Hkv) != g:
                continue
            for r0 in range(t0, S, row_block):
                r1 = min(S, r0 + row_block)
                ts = np.arange(r0, r1)
                Q, dO = _as_f64(q[b, h, r0:r1]), _as_f64(dout[b, h, r0:r1])
                kmax = r1 if causal else S
                s = scale * (Q @ K[:kmax].T)                       # [rows, kmax]
                if causal:
                    s = np.where(np.arange(kmax)[None, :] <= ts[:, None], s, -np.inf)
                p = np.exp(s - s.max(axis=1, keepdims=True))
                p /= p.sum(axis=1, keepdims=True)
                delta = np.sum(dO * (p @ V[:kmax]), axis=1)         # <dO_t, O_t>
                for n, u in zip(idxs, us):
                    if u >= kmax:
                        continue
                    pu = p[:, u]                                    # column u of P (0 where t < u)
                    dS_col = pu * (dO @ V[u] - delta)               # column u of dS
                    dk[n] += scale * (dS_col @ Q)
                    dv[n] += pu @ dO
    return dk, dv
