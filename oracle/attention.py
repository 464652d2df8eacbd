"""Oracle block-sparse causal attention forward, in float64 (test infrastructure).

Definition followed (see the package docstring for who may call this):

* "Block-Sparse Attention" (ai-model-reference), "Math Or Compute Schema":
  Attention(Q_i, K_i, V_i) = softmax(M_B (.) Q_i K_i^T / sqrt(d_k)) V_i, with
  the block mask applied before the softmax so that only selected
  query-block/key-block regions carry weight.  Reading: a dropped pair gets
  -inf before the softmax (an elementwise product would leave it at score 0
  and still give it weight, contradicting the same section's prose).
* "bsbr", "Solution": inside a chunk, softmax attention under the within-chunk
  causal mask M_in; BF1 (section 3.1) has the self block read causally.  The
  causal convention includes the token itself (u <= t).
* The scale is a parameter; every workload uses 1/sqrt(d).

For folded head f (batch*heads), query token t in block i = t // B and key
token u in block j = u // B, u is allowed iff j is kept by (layout head
f % L, block i) and (j < i, or j == i and u <= t).  With s_tu = scale*<q_t,k_u>:
lse_t = log sum_allowed exp(s_tu) and o_t = sum_allowed exp(s_tu - lse_t) v_u,
reading K/V slice f // (heads // kv_heads).  A row with no allowed key has
o_t = 0 and lse_t = -inf.  The last block may be shorter than B.

Three restatements of that one definition:
  forward_dense      -- the full n x n masked score matrix (tiny/medium n).
  forward_sparse     -- the same sums taken only over each row's kept blocks;
                        identical up to rounding order because dropped pairs
                        contribute exp(-inf) = 0.
  forward_bruteforce -- pure Python loops with math.exp (tiny inputs only).
"""
from __future__ import annotations

import math

import numpy as np


def _check(q, k, v):
    if q.ndim != 3 or k.ndim != 3 or v.ndim != 3:
        raise ValueError("q, k, v must be [heads, n, d]")
    heads, n, d = q.shape
    kv_heads = k.shape[0]
    if k.shape != (kv_heads, n, d) or v.shape != (kv_heads, n, d):
        raise ValueError("k, v must be [kv_heads, n, d] with q's n and d")
    if heads % kv_heads:
        raise ValueError("heads must be a multiple of kv_heads")
    return heads, kv_heads, n, d


def token_mask(sets_one_head, n: int, B: int) -> np.ndarray:
    """Boolean n x n mask of allowed (t, u) pairs for one layout head."""
    nb = len(sets_one_head)
    mb = np.zeros((nb, nb), dtype=bool)
    for i, row in enumerate(sets_one_head):
        for j in row:
            mb[i, j] = True
    blk = np.arange(n) // B
    allowed = mb[blk[:, None], blk[None, :]]
    causal = np.arange(n)[None, :] <= np.arange(n)[:, None]
    return allowed & causal


def _softmax_rows(s: np.ndarray):
    """Max-subtracted softmax of rows with -inf entries; returns (p, lse)."""
    m = s.max(axis=1, keepdims=True)
    empty = ~np.isfinite(m[:, 0])
    m_safe = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m_safe)
    l = e.sum(axis=1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        p = np.where(l > 0, e / np.where(l > 0, l, 1.0), 0.0)
        lse = np.where(empty, -np.inf, m_safe[:, 0] + np.log(np.where(l[:, 0] > 0, l[:, 0], 1.0)))
    return p, lse


def forward_dense(q, k, v, sets, B: int, scale: float, return_probs: bool = False):
    """Definitional path: dense n x n masked scores for every folded head.

    q: [heads, n, d], k/v: [kv_heads, n, d] (any float dtype; computed in fp64);
    sets: ``sets[h][i]`` kept blocks of layout head h.  Returns (o, lse[, probs]).
    """
    heads, kv_heads, n, d = _check(q, k, v)
    g = heads // kv_heads
    L = len(sets)
    o = np.zeros((heads, n, d), dtype=np.float64)
    lse = np.zeros((heads, n), dtype=np.float64)
    probs = [] if return_probs else None
    masks = {}
    for f in range(heads):
        lh = f % L
        if lh not in masks:
            masks[lh] = token_mask(sets[lh], n, B)
        mask = masks[lh]
        qf = np.asarray(q[f], dtype=np.float64)
        kf = np.asarray(k[f // g], dtype=np.float64)
        vf = np.asarray(v[f // g], dtype=np.float64)
        s = scale * (qf @ kf.T)
        s = np.where(mask, s, -np.inf)
        p, lse[f] = _softmax_rows(s)
        o[f] = p @ vf
        if return_probs:
            probs.append(p)
    return (o, lse, probs) if return_probs else (o, lse)


def forward_block_rows(q, k, v, sets, B: int, scale: float, f: int, i: int):
    """Support-restricted path for one (folded head f, query block i).

    Gathers the kept key blocks' rows, scores them in fp64, applies the causal
    mask inside the diagonal block and normalises.  Returns (o [rows, d],
    lse [rows]) for tokens i*B .. min(n, (i+1)*B) - 1.
    """
    heads, kv_heads, n, d = _check(q, k, v)
    g = heads // kv_heads
    L = len(sets)
    t0, t1 = i * B, min(n, (i + 1) * B)
    kept = sorted(sets[f % L][i])
    rows = t1 - t0
    if not kept:
        return np.zeros((rows, d)), np.full(rows, -np.inf)
    keys = np.concatenate([np.arange(j * B, min(n, (j + 1) * B)) for j in kept])
    qf = np.asarray(q[f, t0:t1], dtype=np.float64)
    kf = np.asarray(k[f // g][keys], dtype=np.float64)
    vf = np.asarray(v[f // g][keys], dtype=np.float64)
    s = scale * (qf @ kf.T)
    t = np.arange(t0, t1)[:, None]
    u = keys[None, :]
    allowed = (u // B < i) | (u <= t)
    s = np.where(allowed, s, -np.inf)
    p, lse = _softmax_rows(s)
    return p @ vf, lse


def forward_sparse(q, k, v, sets, B: int, scale: float, items=None):
    """Support-restricted path over every (head, block), or over ``items``.

    With ``items`` (a list of (f, i)), returns {(f, i): (o_rows, lse_rows)};
    otherwise full (o [heads, n, d], lse [heads, n]) arrays.
    """
    heads, kv_heads, n, d = _check(q, k, v)
    nb = -(-n // B)
    if items is not None:
        return {(f, i): forward_block_rows(q, k, v, sets, B, scale, f, i) for f, i in items}
    o = np.zeros((heads, n, d), dtype=np.float64)
    lse = np.zeros((heads, n), dtype=np.float64)
    for f in range(heads):
        for i in range(nb):
            ob, lb = forward_block_rows(q, k, v, sets, B, scale, f, i)
            o[f, i * B:i * B + ob.shape[0]] = ob
            lse[f, i * B:i * B + ob.shape[0]] = lb
    return o, lse


def forward_bruteforce(q, k, v, sets, B: int, scale: float):
    """Pure-Python triple loop (math.exp, no NumPy arithmetic); tiny inputs only."""
    heads, kv_heads, n, d = _check(q, k, v)
    g = heads // kv_heads
    L = len(sets)
    ql, kl, vl = q.tolist(), k.tolist(), v.tolist()
    o = [[[0.0] * d for _ in range(n)] for _ in range(heads)]
    lse = [[0.0] * n for _ in range(heads)]
    for f in range(heads):
        kv = f // g
        rows = sets[f % L]
        for t in range(n):
            i = t // B
            scores = []
            for u in range(n):
                j = u // B
                if j in rows[i] and (j < i or u <= t):
                    dot = 0.0
                    for c in range(d):
                        dot += ql[f][t][c] * kl[kv][u][c]
                    scores.append((u, scale * dot))
            if not scores:
                lse[f][t] = -math.inf
                continue
            m = max(s for _, s in scores)
            z = sum(math.exp(s - m) for _, s in scores)
            lse[f][t] = m + math.log(z)
            for u, s in scores:
                w = math.exp(s - m) / z
                for c in range(d):
                    o[f][t][c] += w * vl[kv][u][c]
    return np.array(o), np.array(lse)
