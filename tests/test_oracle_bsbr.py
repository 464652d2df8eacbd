"""Pins for the BSBR retrieval oracle (CPU only).

* Token-level brute force with pure Python loops: o_t = sum_{c' < c} A_cc'
  sum_{u in c'} <q_t, k_u> v_u, the meta weights from explicit sums and
  math.exp -- no chunk state is formed, so a transposed or mis-summed state,
  a wrong chunk mask or a wrong pooling fails it (ragged ends, GQA heads).
* Closed form at scale 0: the meta softmax is uniform, so the term is linear
  attention over the earlier chunks' tokens divided by the chunk index.
* Causality at chunk level; chunk 0 retrieves nothing; a single chunk (B >= n)
  reduces the whole output to dense causal attention (torch's
  scaled_dot_product_attention as the library routine).
* Planted mistakes (an inclusive chunk mask, a transposed state) fail these
  pins.
"""
import math

import numpy as np
import pytest
import torch

from oracle import bsbr as BS
from block_sparse_long_bsa_b200 import inputs


def _rand(heads, kv_heads, n, d, seed=0):
    q, k, v = inputs.qkv_bits(heads, kv_heads, n, d, seeds=(seed, seed + 1, seed + 2))
    return tuple(inputs.bf16_bits_to_f64(x) for x in (q, k, v))


def _brute(q, k, v, B, scale):
    heads, n, d = q.shape
    kv = k.shape[0]
    g = heads // kv
    nc = -(-n // B)
    out = np.zeros((heads, n, d))
    for f in range(heads):
        kh = f // g
        R, H = [], []
        for c in range(nc):
            toks = range(c * B, min(n, (c + 1) * B))
            R.append([sum(q[f, t, x] for t in toks) / len(toks) for x in range(d)])
            H.append([sum(k[kh, t, x] for t in toks) / len(toks) for x in range(d)])
        for c in range(1, nc):
            a = [scale * sum(R[c][x] * H[cp][x] for x in range(d)) for cp in range(c)]
            m = max(a)
            e = [math.exp(z - m) for z in a]
            z = sum(e)
            for t in range(c * B, min(n, (c + 1) * B)):
                acc = [0.0] * d
                for cp in range(c):
                    w = e[cp] / z
                    for u in range(cp * B, (cp + 1) * B):
                        s = sum(q[f, t, x] * k[kh, u, x] for x in range(d))
                        for x in range(d):
                            acc[x] += w * s * v[kh, u, x]
                out[f, t] = acc
    return out


@pytest.mark.parametrize("heads,kv,n,B,d", [(2, 1, 21, 4, 3), (4, 2, 19, 5, 4), (1, 1, 16, 4, 2)])
def test_matches_token_level_brute_force(heads, kv, n, B, d):
    q, k, v = _rand(heads, kv, n, d, seed=3)
    scale = 0.6
    np.testing.assert_allclose(BS.retrieval(q, k, v, B, scale), _brute(q, k, v, B, scale),
                               rtol=1e-11, atol=1e-11)


def test_scale_zero_is_linear_attention_over_earlier_chunks():
    heads, kv, n, B, d = 2, 2, 64, 8, 4
    q, k, v = _rand(heads, kv, n, d, seed=5)
    got = BS.retrieval(q, k, v, B, 0.0)
    for f in range(heads):
        for t in range(n):
            c = t // B
            want = np.zeros(d) if c == 0 else q[f, t] @ (k[f, :c * B].T @ v[f, :c * B]) / c
            np.testing.assert_allclose(got[f, t], want, rtol=1e-12, atol=1e-12)


def test_chunk_level_causality_and_chunk_zero():
    heads, kv, n, B, d = 2, 1, 48, 8, 4
    q, k, v = _rand(heads, kv, n, d, seed=7)
    base = BS.retrieval(q, k, v, B, 0.5)
    assert np.all(base[:, :B] == 0)
    rng = np.random.default_rng(0)
    c = 3
    # anything in later chunks leaves chunks <= c unchanged
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[:, (c + 1) * B:] += rng.standard_normal(q2[:, (c + 1) * B:].shape)
    k2[:, (c + 1) * B:] += rng.standard_normal(k2[:, (c + 1) * B:].shape)
    v2[:, (c + 1) * B:] += rng.standard_normal(v2[:, (c + 1) * B:].shape)
    np.testing.assert_array_equal(BS.retrieval(q2, k2, v2, B, 0.5)[:, :(c + 1) * B], base[:, :(c + 1) * B])
    # chunk c's own keys and values only reach later chunks
    k3, v3 = k.copy(), v.copy()
    k3[:, c * B:(c + 1) * B] += 1.0
    v3[:, c * B:(c + 1) * B] -= 1.0
    after = BS.retrieval(q, k3, v3, B, 0.5)
    np.testing.assert_array_equal(after[:, :(c + 1) * B], base[:, :(c + 1) * B])
    assert np.abs(after[:, (c + 1) * B:] - base[:, (c + 1) * B:]).max() > 1e-3


def test_planted_mistakes_fail_the_pins():
    heads, kv, n, B, d = 1, 1, 20, 4, 3
    q, k, v = _rand(heads, kv, n, d, seed=9)
    brute = _brute(q, k, v, B, 0.7)
    # a transposed state (V^T K instead of K^T V)
    F, H = BS.chunk_states(k, v, B)
    A = BS.meta_weights(q, H, B, 0.7, 1)
    wrong = np.zeros_like(brute)
    for c in range(1, -(-n // B)):
        S = np.tensordot(A[0, c, :c], np.transpose(F[0, :c], (0, 2, 1)), axes=(0, 0))
        wrong[0, c * B:(c + 1) * B] = q[0, c * B:(c + 1) * B] @ S
    assert np.abs(wrong - brute).max() > 1e-3
    # an inclusive chunk mask (c' <= c) lets chunk c's own values in
    incl = np.zeros_like(brute)
    R = np.stack([q[0, c * B:(c + 1) * B].mean(axis=0) for c in range(-(-n // B))])
    for c in range(-(-n // B)):
        s = 0.7 * (R[c] @ H[0, :c + 1].T)
        w = np.exp(s - s.max())
        w /= w.sum()
        incl[0, c * B:(c + 1) * B] = q[0, c * B:(c + 1) * B] @ np.tensordot(w, F[0, :c + 1], axes=(0, 0))
    v2 = v.copy()
    v2[0, 8:12] += 1.0
    F2, _ = BS.chunk_states(k, v2, B)
    incl2 = np.zeros_like(brute)
    for c in range(-(-n // B)):
        s = 0.7 * (R[c] @ H[0, :c + 1].T)
        w = np.exp(s - s.max())
        w /= w.sum()
        incl2[0, c * B:(c + 1) * B] = q[0, c * B:(c + 1) * B] @ np.tensordot(w, F2[0, :c + 1], axes=(0, 0))
    assert np.abs(incl2[0, 8:12] - incl[0, 8:12]).max() > 1e-3      # the causality pin would fail
    assert np.abs(incl - brute).max() > 1e-3


def test_single_chunk_is_dense_causal_attention():
    heads, kv, n, d = 4, 2, 40, 8
    q, k, v = _rand(heads, kv, n, d, seed=11)
    scale = 1.0 / math.sqrt(d)
    o, lse = BS.bsbr_output(q, k, v, 64, scale)
    g = heads // kv
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k).repeat_interleave(g, 0)[None],
        torch.from_numpy(v).repeat_interleave(g, 0)[None], is_causal=True, scale=scale)[0].numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)
