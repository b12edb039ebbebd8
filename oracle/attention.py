"""fp64 CPU oracle for exact (ring) attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or
execute this module: only the tests, the package smoke check and the CPU
baseline leg of the benchmark use it. It shares no code with the CUDA path.

Sources (the RingAttention pages):
  [DEF]  FlashAttention video summary (aitrends), chapter "basic attention
         computation": scores = Q K^T, subtract the row maximum, softmax, weight V.
  [EQ]   RingAttention deep-architecture article (techknowgenie), section 3
         "rigorous derivation of blockwise online softmax": S_ik = Q_i K_k^T / sqrt(d),
         m_block = rowmax(S_ik), m_new = max(m_old, m_block), alpha = exp(m_old - m_new),
         beta = exp(m_block - m_new), P_curr = exp(S_ik - m_block),
         l_new = l_old*alpha + rowsum(P_curr)*beta, O_new = O_old*alpha + (P_curr V_k)*beta,
         O_final = O / l_final.
  [RING] same article, section 2 "core principle": Q_i stays on device i; KV
         blocks move to (i+1) mod P, so at ring step s device i holds block (i-s) mod P;
         section 5 code listing: step 0 uses the device's own KV, P steps in total.
  [MASK] same article, section 7 "causal attention with striped attention": a
         decoder attends to past tokens; striped layout deals tokens round-robin,
         token t on shard t mod P.
  [ZIG]  RingAttention newsletter (cmlonder), section "claim and reality": striped or
         zigzag schedules counter the causal load imbalance of the ring. The page
         names zigzag without defining it; the plainest reading taken here cuts the
         sequence into 2P equal chunks and gives shard i chunks i and 2P-1-i.

Readings where the pages are silent:
  * lse = m + ln(l): natural log, in units of the scaled scores.
  * The causal diagonal is inclusive: key u is allowed for query t iff u <= t.
  * GQA: query head h reads kv head h // (Hq // Hkv).
  * Layout and P only change the schedule: ``attention_reference`` has neither.
  * A block row with no allowed key (m_block = -inf) contributes nothing; with
    m_old = -inf the rescale factor is 0, never exp(nan).

All arithmetic is fp64 on the exact values of the (already rounded) inputs.
"""
from __future__ import annotations

import math
from typing import Iterable, Sequence

import numpy as np

NEG_INF = -math.inf


# --------------------------------------------------------------------------------------
# small pieces (kept separate so tests can plant a mistake in exactly one of them)
# --------------------------------------------------------------------------------------

def kv_head(h: int, Hq: int, Hkv: int) -> int:
    """Query head h reads kv head h // (Hq/Hkv) (consecutive groups)."""
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return h // (Hq // Hkv)


def allowed_keys(t, S: int, causal: bool):
    """Number of keys query token t may see: keys 0..t (inclusive diagonal) or all S.

    Works on ints and on integer arrays of tokens; key u is allowed iff u < allowed_keys(t).
    """
    if causal:
        return t + 1
    return S if np.isscalar(t) else np.full_like(t, S)


def shard_tokens(S: int, P: int, layout: str, i: int) -> np.ndarray:
    """Global token ids held by shard i, in local order.

    contiguous: tokens [i*S/P, (i+1)*S/P); striped: tokens a*P + i for a = 0..S/P-1;
    zigzag [ZIG]: with chunks of C = S/(2P) tokens, chunk i then chunk 2P-1-i.
    """
    if S % P != 0:
        raise ValueError("S must be a multiple of P")
    Sq = S // P
    a = np.arange(Sq, dtype=np.int64)
    if layout == "contiguous":
        return i * Sq + a
    if layout == "striped":
        return a * P + i
    if layout == "zigzag":
        if S % (2 * P) != 0:
            raise ValueError("zigzag needs S to be a multiple of 2P")
        C = S // (2 * P)
        c = np.arange(C, dtype=np.int64)
        return np.concatenate([i * C + c, (2 * P - 1 - i) * C + c])
    raise ValueError(f"unknown layout {layout!r}")


def softmax_stats(s: np.ndarray):
    """Max-subtracted exponentials of score rows [DEF]: (p, m, l) with p = exp(s - m),
    m = row max, l = row sum of p. Masked entries are -inf and give p = 0."""
    m = np.max(s, axis=-1, keepdims=True)
    p = np.exp(s - m)
    l = np.sum(p, axis=-1, keepdims=True)
    return p, m, l


def softmax_row(s: np.ndarray) -> tuple[np.ndarray, float]:
    """Softmax of one score vector; returns (p / l, m + ln l)."""
    p, m, l = softmax_stats(s)
    return p / l, float(m[0] + math.log(l[0]))


def _as_f64(x) -> np.ndarray:
    """Exact fp64 copy of a torch tensor (fp32/bf16 -> fp64 is exact) or array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------------------
# the plain definition
# --------------------------------------------------------------------------------------

def attention_rows(q, k, v, rows: Iterable[tuple[int, int, int]], causal: bool, scale: float,
                   chunk: int = 32) -> tuple[np.ndarray, np.ndarray]:
    """Exact attention for selected query rows, one materialised score row each.

    q [B,Hq,S,D], k/v [B,Hkv,S,D] (torch or numpy, any float dtype).
    rows: (b, h, t) triples. Returns O [n, D] and lse [n] in fp64, in ``rows`` order.
    For each row: s_u = scale * <q[b,h,t], k[b,g,u]> over the allowed keys u,
    then the max-subtracted softmax [DEF] weights v[b,g,u].
    """
    rows = list(rows)
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    out = np.zeros((len(rows), D), dtype=np.float64)
    lse = np.zeros(len(rows), dtype=np.float64)
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
        Qh = q[b, h]
        for c0 in range(0, len(idxs), chunk):
            part = idxs[c0:c0 + chunk]
            ts = [rows[n][2] for n in part]
            qs = _as_f64(Qh[ts])                                  # [n, D]
            kmax = max(allowed_keys(t, S, causal) for t in ts)
            s = scale * (qs @ K[:kmax].T)                          # [n, kmax]
            for r, (n, t) in enumerate(zip(part, ts)):
                na = allowed_keys(t, S, causal)
                p, lse[n] = softmax_row(s[r, :na])
                out[n] = p @ V[:na]
    return out, lse


def attention_reference(q, k, v, causal: bool, scale: float, row_block: int = 256
                        ) -> tuple[np.ndarray, np.ndarray]:
    """Exact attention for every row: O [B,Hq,S,D], lse [B,Hq,S] in fp64.

    Score rows are formed a block of rows at a time with one matrix product,
    then each row is masked (keys u <= t when causal) and soft-maxed [DEF].
    """
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    O = np.zeros((B, Hq, S, D), dtype=np.float64)
    L = np.zeros((B, Hq, S), dtype=np.float64)
    for b in range(B):
        for g in range(Hkv):
            K = _as_f64(k[b, g])
            V = _as_f64(v[b, g])
            for h in range(Hq):
                if kv_head(h, Hq, Hkv) != g:
                    continue
                Q = _as_f64(q[b, h])
                for r0 in range(0, S, row_block):
                    r1 = min(S, r0 + row_block)
                    kmax = r1 if causal else S
                    s = scale * (Q[r0:r1] @ K[:kmax].T)          # [rows, kmax]
                    lim = allowed_keys(np.arange(r0, r1), S, causal)
                    s = np.where(np.arange(kmax)[None, :] < lim[:, None], s, NEG_INF)
                    p, m, l = softmax_stats(s)
                    O[b, h, r0:r1] = (p @ V[:kmax]) / l
                    L[b, h, r0:r1] = (m + np.log(l))[:, 0]
    return O, L


# --------------------------------------------------------------------------------------
# the ring recurrence, as the pages state it
# --------------------------------------------------------------------------------------

def block_allowed(tq: np.ndarray, tk: np.ndarray, causal: bool) -> np.ndarray:
    """Mask of a (query shard, key shard) block on global token order [MASK]."""
    return tk[None, :] < allowed_keys(tq, 0 if causal else 1 << 62, causal)[:, None]


def ring_attention_online(q, k, v, P: int, causal: bool, layout: str, scale: float
                          ) -> tuple[np.ndarray, np.ndarray]:
    """Blockwise online softmax over P shards in ring order, in fp64.

    For each query shard i, the state (m = -inf, l = 0, O = 0) folds KV shard
    j = (i - s) mod P at ring step s = 0..P-1 [RING] with the alpha/beta update
    of [EQ], then O_final = O / l and lse = m + ln l. Outputs are scattered back
    to natural token order: O [B,Hq,S,D], lse [B,Hq,S].
    """
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    O_out = np.zeros((B, Hq, S, D), dtype=np.float64)
    L_out = np.zeros((B, Hq, S), dtype=np.float64)
    shards = [shard_tokens(S, P, layout, i) for i in range(P)]
    for b in range(B):
        for h in range(Hq):
            g = kv_head(h, Hq, Hkv)
            Qa, Ka, Va = _as_f64(q[b, h]), _as_f64(k[b, g]), _as_f64(v[b, g])
            for i in range(P):
                tq = shards[i]
                Qi = Qa[tq]
                n = tq.size
                m = np.full(n, NEG_INF)
                l = np.zeros(n)
                O = np.zeros((n, D))
                for s in range(P):
                    j = (i - s) % P
                    tk = shards[j]
                    Sik = scale * (Qi @ Ka[tk].T)
                    Sik = np.where(block_allowed(tq, tk, causal), Sik, NEG_INF)
                    m_block = Sik.max(axis=1)
                    m_new = np.maximum(m, m_block)
                    # a row whose old and new maxima are both -inf has seen no key yet:
                    # its factors are 0 (nothing to keep, nothing to add)
                    live = np.isfinite(m_new)
                    alpha = np.where(np.isfinite(m), np.exp(m - np.where(live, m_new, 0.0)), 0.0)
                    has_block = np.isfinite(m_block)
                    beta = np.where(has_block, np.exp(np.where(has_block, m_block, 0.0)
                                                      - np.where(live, m_new, 0.0)), 0.0)
                    sub = np.where(has_block, m_block, 0.0)[:, None]
                    P_curr = np.where(np.isfinite(Sik), np.exp(Sik - sub), 0.0)
                    l = l * alpha + P_curr.sum(axis=1) * beta
                    O = O * alpha[:, None] + (P_curr @ Va[tk]) * beta[:, None]
                    m = m_new
                O_out[b, h, tq] = O / l[:, None]
                L_out[b, h, tq] = m + np.log(l)
    return O_out, L_out


# --------------------------------------------------------------------------------------
# combining normalised partial results
# --------------------------------------------------------------------------------------

def merge_partials(o_parts: Sequence[np.ndarray], lse_parts: Sequence[np.ndarray]
                   ) -> tuple[np.ndarray, np.ndarray]:
    """Combine normalised partials (O_k = softmax over key subset k applied to V, lse_k).

    With L = ln sum_k exp(lse_k), the full result is O = sum_k exp(lse_k - L) O_k:
    the alpha/beta algebra of [EQ] applied to states whose l has already been
    divided out. Parts with lse = -inf are empty and get weight 0; if every part
    is empty the result is O = 0, lse = -inf.
    o_parts: n arrays [..., D]; lse_parts: n arrays [...] (same leading shape).
    """
    lse_stack = np.stack([_as_f64(x) for x in lse_parts])          # [n, rows]
    o_stack = np.stack([_as_f64(x) for x in o_parts])              # [n, rows, D]
    mx = lse_stack.max(axis=0)                                     # [rows]
    empty = ~np.isfinite(mx)
    mx_safe = np.where(empty, 0.0, mx)
    w = np.where(np.isfinite(lse_stack), np.exp(lse_stack - mx_safe[None, :]), 0.0)
    tot = w.sum(axis=0)
    lse = np.where(empty, NEG_INF, mx_safe + np.log(np.where(empty, 1.0, tot)))
    wn = np.where(empty[None, :], 0.0, w / np.where(empty, 1.0, tot)[None, :])
    O = np.sum(wn[..., None] * o_stack, axis=0)
    return O, lse


def attention_keyset(q, k, v, key_mask: np.ndarray, scale: float
                     ) -> tuple[np.ndarray, np.ndarray]:
    """Attention of every query row over an arbitrary allowed-key mask [B,Hq,S,S].

    Rows with no allowed key return O = 0 and lse = -inf (an empty partial).
    Used to build partials for the merge pins.
    """
    B, Hq, S, D = q.shape
    Hkv = k.shape[1]
    O = np.zeros((B, Hq, S, D))
    L = np.full((B, Hq, S), NEG_INF)
    for b in range(B):
        for h in range(Hq):
            g = kv_head(h, Hq, Hkv)
            Q, K, V = _as_f64(q[b, h]), _as_f64(k[b, g]), _as_f64(v[b, g])
            s = scale * (Q @ K.T)
            for t in range(S):
                sel = key_mask[b, h, t]
                if not sel.any():
                    continue
                p, L[b, h, t] = softmax_row(s[t, sel])
                O[b, h, t] = p @ V[sel]
    return O, L
