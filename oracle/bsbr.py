"""Oracle of BSBR's between-chunk retrieval term, in float64 (test
infrastructure; only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU legs may call it).

Definition followed: "bsbr" (jvboid.dev/projects/bsbr), section "Solution".
The sequence is cut into chunks of B tokens.  Inside a chunk, softmax
attention under the within-chunk causal mask (the block-diagonal layout of
``oracle.attention``).  Between chunks, retrieval: each chunk is compressed
into a state F_c, the flattened K_c^T V_c of its tokens; meta queries R and
meta keys H act at chunk granularity, M_out is the causal mask over chunks,
and the chunk-level result is broadcast back over the B tokens of its chunk
and read by the query.  The output is the sum of the two terms.

Readings where the page is silent (each listed in the design notes):
  * R_c and H_c are the means of q and k over the tokens of chunk c (the page
    does not define them; mean pooling is the plainest meta query/key of a
    chunk).  R_c pools every token of chunk c, so the retrieval weights of a
    token depend on its own chunk's queries (never on its keys or values).
  * M_out keeps strictly earlier chunks (c' < c): a chunk's own state holds
    keys and values of its later tokens, and its tokens are covered exactly
    by the within-chunk term.  Chunk 0 retrieves nothing (its term is 0).
  * The meta scores carry the same scale as the token scores: a_cc' =
    scale <R_c, H_c'>, softmax over c' < c.
  * "Q (.) ... F.repeat(B)": token t of chunk c reads the retrieved d x d
    state S_c = sum_c' A_cc' F_c' with its query, o_t = q_t S_c (the state is
    K^T V, so this is how a query reads it; an elementwise product of a
    d-vector with a d^2-vector has no meaning).
  * States are not normalised (K_c^T V_c as written); a partial last chunk
    pools and sums over the tokens it has.
Grouped-query heads: query head f reads key/value head f // (heads // kv_heads)
for H and F; R is per query head.
"""
from __future__ import annotations

import numpy as np

from oracle.attention import _check, forward_dense


def n_chunks(n: int, B: int) -> int:
    return -(-n // B)


def chunk_states(k, v, B: int):
    """F [kv_heads, chunks, d, d] = K_c^T V_c and H [kv_heads, chunks, d] =
    mean of k over chunk c."""
    kv_heads, n, d = k.shape
    nc = n_chunks(n, B)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    F = np.zeros((kv_heads, nc, d, d))
    H = np.zeros((kv_heads, nc, d))
    for g in range(kv_heads):
        for c in range(nc):
            kc = k[g, c * B:(c + 1) * B]
            vc = v[g, c * B:(c + 1) * B]
            F[g, c] = kc.T @ vc
            H[g, c] = kc.mean(axis=0)
    return F, H


def meta_weights(q, H, B: int, scale: float, group: int):
    """A [heads, chunks, chunks]: softmax over c' < c of scale <R_c, H_c'>,
    R_c the mean of q over chunk c; row 0 (no earlier chunk) is all zeros."""
    heads, n, d = q.shape
    nc = n_chunks(n, B)
    q = np.asarray(q, dtype=np.float64)
    A = np.zeros((heads, nc, nc))
    for f in range(heads):
        R = np.stack([q[f, c * B:(c + 1) * B].mean(axis=0) for c in range(nc)])
        s = scale * (R @ H[f // group].T)
        for c in range(1, nc):
            row = s[c, :c]
            e = np.exp(row - row.max())
            A[f, c, :c] = e / e.sum()
    return A


def retrieval(q, k, v, B: int, scale: float):
    """The between-chunk term o_ret [heads, n, d]: o_t = q_t S_c(t),
    S_c = sum_{c' < c} A_cc' F_c'."""
    heads, kv_heads, n, d = _check(q, k, v)
    group = heads // kv_heads
    nc = n_chunks(n, B)
    F, H = chunk_states(k, v, B)
    A = meta_weights(q, H, B, scale, group)
    q = np.asarray(q, dtype=np.float64)
    out = np.zeros((heads, n, d))
    for f in range(heads):
        g = f // group
        for c in range(1, nc):
            S = np.tensordot(A[f, c, :c], F[g, :c], axes=(0, 0))
            out[f, c * B:(c + 1) * B] = q[f, c * B:(c + 1) * B] @ S
    return out


def within_chunk_sets(n: int, B: int):
    """The within-chunk term's layout: chunk i keeps only itself."""
    return [[{i} for i in range(n_chunks(n, B))]]


def bsbr_output(q, k, v, B: int, scale: float):
    """(o, lse_in): the full BSBR attention output (within-chunk softmax
    attention plus the retrieval term) and the within-chunk term's lse."""
    n = q.shape[1]
    o_in, lse_in = forward_dense(q, k, v, within_chunk_sets(n, B), B, scale)
    return o_in + retrieval(q, k, v, B, scale), lse_in
