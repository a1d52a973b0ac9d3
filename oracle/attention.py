"""Plain float64 attention over a paged KV cache (test oracle; see package doc).

What is computed (POD-Attention explainer, "Why this problem is worth solving"):
for each query token, attention is a weighted combination of the keys and values
of all earlier tokens, which live in the KV cache.  Prefill processes a chunk of
prompt tokens at once (hybrid batching = chunked prefill, "What people did");
decode processes one new token per request and reads that request's whole cache.

Readings where the cited sources are silent (the plainest one in each case):
  * weights are softmax(scale * q . k) in the natural base;
  * causal alignment is bottom-right: chunk row i sits at absolute position C+i
    and sees keys 0..C+i (the chunk continues a prompt of C earlier tokens whose
    K/V, together with the chunk's own, are already in the cache);
  * a decode query sees all L_r tokens of its request;
  * GQA: query head h reads kv head h // (Hq / Hkv);
  * paged layout: token j of a request is slot j % 16 of block table entry j // 16;
  * inputs are the bf16 values upcast exactly to float64.

Split-KV (POD-Attention explainer, "Cap prefill splitting to avoid contention",
FlashDecoding-style) computes a partial result per key range; the ranges are
combined by a log-sum-exp merge (the PAT catalogue record merges its per-split
results with online softmax).  ``attend_partial`` / ``lse_merge`` state that merge.
"""
from __future__ import annotations

import math
from typing import List, Sequence, Tuple

import numpy as np

PAGE = 16


def gather_tokens(pool: np.ndarray, bt_row: np.ndarray, length: int, kv_head: int) -> np.ndarray:
    """Rows 0..length-1 of one request's K (or V) for one kv head, as float64 [length, d].

    ``pool`` is [num_blocks, Hkv, 16, d], either bf16 bit patterns (uint16) or
    floats; token j lives in block bt_row[j // 16], slot j % 16.  Only the
    gathered tokens are upcast."""
    d = pool.shape[-1]
    npages = (length + PAGE - 1) // PAGE
    blocks = np.asarray(bt_row[:npages], dtype=np.int64)
    pages = pool[blocks, kv_head]                       # [npages, 16, d]
    return _as_f64(pages.reshape(npages * PAGE, d)[:length])


def attend_rows(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float, limits: Sequence[int]) -> np.ndarray:
    """Row i of q attends to keys 0..limits[i]-1 of K/V: softmax(scale q K^T) V.

    q [n, d], K/V [L, d], all float64; a numerically stable softmax (row max
    subtracted before exponentiation)."""
    s = (q @ K.T) * scale
    L = K.shape[0]
    lim = np.asarray(limits, dtype=np.int64)
    mask = np.arange(L)[None, :] >= lim[:, None]
    s = np.where(mask, -np.inf, s)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    return (p @ V) / p.sum(axis=1, keepdims=True)


def _as_f64(bits_or_f: np.ndarray) -> np.ndarray:
    if bits_or_f.dtype == np.uint16:
        return (bits_or_f.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return np.asarray(bits_or_f, dtype=np.float64)


def attend_decode(q_dec, k_pool, v_pool, block_table, kv_lens, scale: float, num_kv_heads: int,
                  requests=None, first_row: int = 1) -> np.ndarray:
    """Decode attention.  q_dec [B, Hq, d]; row first_row + r of block_table /
    kv_lens is request r (the rows before it belong to the prefill requests).

    Returns float64 [B, Hq, d] (or [len(requests), Hq, d] for a subset)."""
    q = _as_f64(q_dec)
    kp, vp = k_pool, v_pool
    B, Hq, d = q.shape
    g = Hq // num_kv_heads
    reqs = range(B) if requests is None else list(requests)
    out = np.empty((len(reqs), Hq, d), dtype=np.float64)
    for o, r in enumerate(reqs):
        L = int(kv_lens[first_row + r])
        for kvh in range(num_kv_heads):
            K = gather_tokens(kp, block_table[first_row + r], L, kvh)
            V = gather_tokens(vp, block_table[first_row + r], L, kvh)
            hs = slice(kvh * g, (kvh + 1) * g)
            out[o, hs] = attend_rows(q[r, hs], K, V, scale, [L] * g)
    return out


def attend_prefill(q_pre, k_pool, v_pool, block_table, prior_ctx: int, scale: float, num_kv_heads: int,
                   rows=None, bt_row: int = 0) -> np.ndarray:
    """Causal chunked-prefill attention for the request in block_table row bt_row.

    q_pre [P, Hq, d]; chunk row i sees keys 0..C+i.  Returns float64 [P, Hq, d]
    (or [len(rows), Hq, d] for a subset of chunk rows)."""
    q = _as_f64(q_pre)
    kp, vp = k_pool, v_pool
    P, Hq, d = q.shape
    C = int(prior_ctx)
    g = Hq // num_kv_heads
    sel = np.arange(P) if rows is None else np.asarray(list(rows), dtype=np.int64)
    out = np.empty((len(sel), Hq, d), dtype=np.float64)
    if len(sel) == 0:
        return out
    L = C + int(sel.max()) + 1
    limits = C + sel + 1
    for kvh in range(num_kv_heads):
        K = gather_tokens(kp, block_table[bt_row], L, kvh)
        V = gather_tokens(vp, block_table[bt_row], L, kvh)
        for hh in range(g):
            h = kvh * g + hh
            out[:, h] = attend_rows(q[sel, h], K, V, scale, limits)
    return out


def attend_prefill_batched(q_pre, k_pool, v_pool, block_table, qo_lens, kv_lens, scale: float,
                           num_kv_heads: int, rows=None) -> np.ndarray:
    """Several chunked-prefill requests in one hybrid batch (the FlashInfer PR
    "Limit kv split when prefill tokens <= 1536" times such a "Batched POD
    Attention" next to the one-prefill POD): request i owns block_table row i, its P_i = qo_lens[i] query
    rows follow those of requests 0..i-1 in q_pre [sum P_i, Hq, d], and its chunk
    continues C_i = kv_lens[i] - P_i earlier tokens.  Each request is the single
    chunked prefill above.  Returns float64 [sum P_i, Hq, d] (or the rows listed,
    indexed into the concatenation)."""
    q = _as_f64(q_pre)
    total, Hq, d = q.shape
    sel = np.arange(total) if rows is None else np.asarray(list(rows), dtype=np.int64)
    out = np.empty((len(sel), Hq, d), dtype=np.float64)
    start = 0
    for i, (P, KV) in enumerate(zip(qo_lens, kv_lens)):
        P, KV = int(P), int(KV)
        mine = (sel >= start) & (sel < start + P)
        if mine.any():
            local = sel[mine] - start
            out[mine] = attend_prefill(q[start:start + P], k_pool, v_pool, block_table, KV - P, scale,
                                       num_kv_heads, rows=local, bt_row=i)
        start += P
    return out


def attend_partial(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float, k0: int, k1: int) -> Tuple[np.ndarray, np.ndarray]:
    """Attention of q [n, d] over keys k0..k1-1 only.

    Returns (O_s, lse_s): O_s [n, d] normalised over that range and
    lse_s [n] = log(sum_j exp(scale q.k_j)) over the same range (natural log)."""
    s = (q @ K[k0:k1].T) * scale
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    return (p @ V[k0:k1]) / l, (m + np.log(l))[:, 0]


def lse_merge(parts: List[Tuple[np.ndarray, np.ndarray]]) -> np.ndarray:
    """Combine split partials: M = max_s lse_s; O = sum_s e^(lse_s - M) O_s / sum_s e^(lse_s - M)."""
    lses = np.stack([p[1] for p in parts])          # [S, n]
    M = lses.max(axis=0)
    w = np.exp(lses - M)                              # [S, n]
    num = sum(w[s][:, None] * parts[s][0] for s in range(len(parts)))
    return num / w.sum(axis=0)[:, None]


# ---------------------------------------------------------------------------
# Brute force (pure Python loops, tiny inputs only).
# ---------------------------------------------------------------------------

def _brute_one(qv: List[float], keys: List[List[float]], vals: List[List[float]], scale: float) -> List[float]:
    scores = []
    for k in keys:
        acc = 0.0
        for a, b in zip(qv, k):
            acc += a * b
        scores.append(acc * scale)
    mx = max(scores)
    ws = [math.exp(s - mx) for s in scores]
    tot = sum(ws)
    d = len(vals[0])
    out = [0.0] * d
    for w, v in zip(ws, vals):
        for c in range(d):
            out[c] += w * v[c]
    return [x / tot for x in out]


def _token(pool, bt_row, j, kvh):
    return [float(x) for x in pool[int(bt_row[j // PAGE]), kvh, j % PAGE, :]]


def attend_brute_decode(q_dec, k_pool, v_pool, block_table, kv_lens, scale: float, num_kv_heads: int,
                        first_row: int = 1) -> np.ndarray:
    q = _as_f64(q_dec)
    kp, vp = _as_f64(k_pool), _as_f64(v_pool)
    B, Hq, d = q.shape
    g = Hq // num_kv_heads
    out = np.zeros((B, Hq, d))
    for r in range(B):
        L = int(kv_lens[first_row + r])
        for h in range(Hq):
            kvh = h // g
            keys = [_token(kp, block_table[first_row + r], j, kvh) for j in range(L)]
            vals = [_token(vp, block_table[first_row + r], j, kvh) for j in range(L)]
            out[r, h] = _brute_one([float(x) for x in q[r, h]], keys, vals, scale)
    return out


def attend_brute_prefill(q_pre, k_pool, v_pool, block_table, prior_ctx: int, scale: float, num_kv_heads: int,
                         bt_row: int = 0) -> np.ndarray:
    q = _as_f64(q_pre)
    kp, vp = _as_f64(k_pool), _as_f64(v_pool)
    P, Hq, d = q.shape
    g = Hq // num_kv_heads
    out = np.zeros((P, Hq, d))
    for i in range(P):
        for h in range(Hq):
            kvh = h // g
            n = prior_ctx + i + 1
            keys = [_token(kp, block_table[bt_row], j, kvh) for j in range(n)]
            vals = [_token(vp, block_table[bt_row], j, kvh) for j in range(n)]
            out[i, h] = _brute_one([float(x) for x in q[i, h]], keys, vals, scale)
    return out
