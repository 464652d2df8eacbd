"""Oracle backward of the block-sparse causal attention forward, in float64
(test infrastructure; only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU legs may call it).

BF1 ("BF1: A Causal Dyadic Sparse-Attention Retrofit for Efficient
Long-Context Transformers", section 4) gates its operator on gradients as well
as on the forward, and its adaptation campaign trains through the route, so
the gradients of o with respect to q, k and v are the ones of the forward's
definition (``oracle.attention``): with P_tu = exp(s_tu - lse_t) over the
allowed pairs (0 elsewhere), s_tu = scale * <q_t, k_u>,

  dV_u = sum_t P_tu dO_t                      (over query rows t reading u)
  dP_tu = <dO_t, v_u>
  D_t = sum_u P_tu dP_tu = <dO_t, o_t>
  dS_tu = P_tu (dP_tu - D_t)
  dQ_t = scale * sum_u dS_tu k_u
  dK_u = scale * sum_t dS_tu q_t

With grouped-query heads, a key/value head's gradients sum over the query
heads that read it.  This follows the softmax's Jacobian written out; the
pins check it against finite differences of the forward and against torch's
autograd of its dense attention on layouts that reduce to it.  A row with no
allowed key (o = 0, lse = -inf) contributes nothing.
"""
from __future__ import annotations

import numpy as np

from oracle.attention import _check, token_mask


def backward_dense(q, k, v, do, sets, B: int, scale: float):
    """(dq, dk, dv) from the full n x n masked probabilities (small n)."""
    heads, kv_heads, n, d = _check(q, k, v)
    g = heads // kv_heads
    L = len(sets)
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    masks = [token_mask(sets[h], n, B) for h in range(L)]
    for f in range(heads):
        kh = f // g
        s = scale * (q[f] @ k[kh].T)
        s = np.where(masks[f % L], s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        live = np.isfinite(m[:, 0])
        e = np.where(live[:, None], np.exp(s - np.where(live[:, None], m, 0.0)), 0.0)
        z = e.sum(axis=1, keepdims=True)
        p = np.where(live[:, None], e / np.where(z > 0, z, 1.0), 0.0)
        o = p @ v[kh]
        dp = do[f] @ v[kh].T
        dd = np.sum(do[f] * o, axis=1, keepdims=True)
        ds = p * (dp - dd)
        dq[f] = scale * (ds @ k[kh])
        dk[kh] += scale * (ds.T @ q[f])
        dv[kh] += p.T @ do[f]
    return dq, dk, dv


def _rows_p(q, k, v, sets, B, scale, f, i):
    """P, allowed keys and o for the rows of (folded head f, query block i)."""
    heads, kv_heads, n, d = _check(q, k, v)
    g = heads // kv_heads
    L = len(sets)
    t0, t1 = i * B, min(n, (i + 1) * B)
    kept = sorted(sets[f % L][i])
    keys = np.concatenate([np.arange(j * B, min(n, (j + 1) * B)) for j in kept]) if kept else np.zeros(0, int)
    qf = np.asarray(q[f, t0:t1], dtype=np.float64)
    kf = np.asarray(k[f // g][keys], dtype=np.float64)
    vf = np.asarray(v[f // g][keys], dtype=np.float64)
    s = scale * (qf @ kf.T)
    t = np.arange(t0, t1)[:, None]
    allowed = (keys[None, :] // B < i) | (keys[None, :] <= t)
    s = np.where(allowed, s, -np.inf)
    m = s.max(axis=1, keepdims=True) if keys.size else np.full((t1 - t0, 1), -np.inf)
    live = np.isfinite(m[:, 0])
    e = np.where(live[:, None], np.exp(s - np.where(live[:, None], m, 0.0)), 0.0)
    z = e.sum(axis=1, keepdims=True)
    p = np.where(live[:, None], e / np.where(z > 0, z, 1.0), 0.0)
    return p, keys, qf, kf, vf, p @ vf


def backward_block_dq(q, k, v, do, sets, B: int, scale: float, f: int, i: int):
    """dQ rows of (folded head f, query block i) over that row's kept blocks."""
    p, keys, qf, kf, vf, o = _rows_p(q, k, v, sets, B, scale, f, i)
    t0 = i * B
    dof = np.asarray(do[f, t0:t0 + p.shape[0]], dtype=np.float64)
    dp = dof @ vf.T
    dd = np.sum(dof * o, axis=1, keepdims=True)
    return scale * ((p * (dp - dd)) @ kf)


def backward_block_dkv(q, k, v, do, sets, B: int, scale: float, kh: int, j: int):
    """dK, dV rows of key/value head kh, key block j: the sum over every query
    head of the group and every query block whose row keeps j."""
    heads, kv_heads, n, d = _check(q, k, v)
    g = heads // kv_heads
    L = len(sets)
    u0, u1 = j * B, min(n, (j + 1) * B)
    dk = np.zeros((u1 - u0, d))
    dv = np.zeros((u1 - u0, d))
    for f in range(kh * g, (kh + 1) * g):
        for i in range(_n_blocks(n, B)):
            if j not in sets[f % L][i]:
                continue
            p, keys, qf, kf, vf, o = _rows_p(q, k, v, sets, B, scale, f, i)
            t0 = i * B
            dof = np.asarray(do[f, t0:t0 + p.shape[0]], dtype=np.float64)
            dp = dof @ vf.T
            dd = np.sum(dof * o, axis=1, keepdims=True)
            ds = p * (dp - dd)
            cols = (keys >= u0) & (keys < u1)
            dk += scale * (ds[:, cols].T @ qf)
            dv += p[:, cols].T @ dof
    return dk, dv


def _n_blocks(n: int, B: int) -> int:
    return -(-n // B)
