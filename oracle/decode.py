"""Oracle decode step over a paged K/V cache, in float64 (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU legs may
call this module; the product path never does.

What a decode step computes ("BF1: A Causal Dyadic Sparse-Attention Retrofit
for Efficient Long-Context Transformers", section 5, selected-page decode: one
new query token per sequence reads the same block route as prefill, over the
cached keys and values; the route is planned once and reused for every token):
for sequence b whose new token sits at position t (block i = t // B), query
head f of that sequence attends to the cached keys u <= t of the key blocks
that block row i of layout head f % L keeps, with the forward's definition
(see ``oracle.attention``): s_u = scale * <q_f, k_u>, lse = log sum exp s_u,
o = sum exp(s_u - lse) v_u.  A row with no allowed key gives o = 0 and
lse = -inf.  This is row t of the forward over the sequence's first t + 1
tokens.

The cache is paged by blocks: page p holds the B consecutive tokens of one
logical key block for every key/value head of a sequence,
``k_cache[p][kv_head][row][d]``, and ``page_table[b][j]`` names the page that
holds logical block j of sequence b.

Readings where the pages are silent: the page size equals the block size B
(the route selects whole blocks, so a selected block is a selected page); the
new token's own key and value are already in the cache when the step runs;
folded heads, as in the forward: ``heads = batch * H`` query rows and
``kv_heads = batch * H_kv`` key/value heads, sequence b owning query rows
b*H .. b*H + H - 1, query head h of a sequence reading its key/value head
h // (H // H_kv).
"""
from __future__ import annotations

import numpy as np


def _softmax_row(s):
    m = np.max(s)
    if not np.isfinite(m):
        return np.zeros_like(s), -np.inf
    e = np.exp(s - m)
    z = e.sum()
    return e / z, m + np.log(z)


def decode_step(q, k_cache, v_cache, page_table, positions, sets, B: int, scale: float):
    """One decode step for every sequence of the batch.

    q: [batch*H, d]; k_cache, v_cache: [pages, H_kv, B, d]; page_table:
    [batch, max_blocks] int; positions: [batch] int; sets: kept-block sets
    ``sets[layout_head][block]`` (as built by ``oracle.layouts``).
    Returns (o [batch*H, d] float64, lse [batch*H] float64).
    """
    q = np.asarray(q, dtype=np.float64)
    heads, d = q.shape
    batch = len(positions)
    if heads % batch:
        raise ValueError("query rows must be a multiple of the batch")
    H = heads // batch
    hkv = k_cache.shape[1]
    if H % hkv:
        raise ValueError("query heads per sequence must be a multiple of its key/value heads")
    g = H // hkv
    L = len(sets)
    o = np.zeros((heads, d))
    lse = np.full(heads, -np.inf)
    for b in range(batch):
        t = int(positions[b])
        i = t // B
        for h in range(H):
            f = b * H + h
            kept = sorted(sets[f % L][i])
            keys, vals, toks = [], [], []
            for j in kept:
                page = int(page_table[b][j])
                rows = np.arange(B)
                tok = j * B + rows
                use = tok <= t                       # causal: only cached tokens up to t
                keys.append(np.asarray(k_cache[page, h // g], dtype=np.float64)[use])
                vals.append(np.asarray(v_cache[page, h // g], dtype=np.float64)[use])
                toks.append(tok[use])
            if not keys:
                continue
            kf = np.concatenate(keys)
            vf = np.concatenate(vals)
            if kf.shape[0] == 0:
                continue
            p, lse[f] = _softmax_row(scale * (kf @ q[f]))
            o[f] = p @ vf
    return o, lse


def pages_from_sequences(k, v, batch: int, B: int, page_order):
    """Scatter contiguous per-sequence K/V into a paged cache.

    k, v: [batch*H_kv, n, d]; page_order: a permutation of range(batch * nb)
    giving, for each (sequence b, block j) in row-major order, the page that
    holds it.  Returns (k_cache, v_cache, page_table) with the layout
    ``decode_step`` reads.  Test helper: it only moves data.
    """
    kvh, n, d = k.shape
    hkv = kvh // batch
    nb = -(-n // B)
    pages = batch * nb
    kc = np.zeros((pages, hkv, B, d), dtype=k.dtype)
    vc = np.zeros((pages, hkv, B, d), dtype=v.dtype)
    table = np.zeros((batch, nb), dtype=np.int32)
    for b in range(batch):
        for j in range(nb):
            p = int(page_order[b * nb + j])
            table[b, j] = p
            r = min(n, (j + 1) * B) - j * B
            for hk in range(hkv):
                kc[p, hk, :r] = k[b * hkv + hk, j * B:j * B + r]
                vc[p, hk, :r] = v[b * hkv + hk, j * B:j * B + r]
    return kc, vc, table
