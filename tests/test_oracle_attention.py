"""Pins for the oracle's attention forward (CPU only).

Pins: reductions to torch's scaled_dot_product_attention / logsumexp (library
routines) for the layouts that collapse to dense causal attention, closed
forms, invariants (row sums, dropped-block and future-token perturbation),
pure-Python brute force on tiny inputs, and agreement between the dense and
support-restricted restatements on every pattern family.
"""
import math

import numpy as np
import pytest
import torch

from oracle import layouts as L
from oracle import attention as A
from block_sparse_long_bsa_b200 import inputs
from block_sparse_long_bsa_b200.workloads import WORKLOADS


def _rand(heads, kv_heads, n, d, seed=0):
    q, k, v = inputs.qkv_bits(heads, kv_heads, n, d, seeds=(seed, seed + 1, seed + 2))
    return inputs.bf16_bits_to_f64(q), inputs.bf16_bits_to_f64(k), inputs.bf16_bits_to_f64(v)


def _all_ones(n, B, heads=1):
    nb = L.n_blocks(n, B)
    return [[set(range(i + 1)) for i in range(nb)] for _ in range(heads)]


def _sdpa_causal(q, k, v, scale):
    heads, kv = q.shape[0], k.shape[0]
    g = heads // kv
    qt = torch.from_numpy(q)[None]
    kt = torch.from_numpy(np.repeat(k, g, axis=0))[None]
    vt = torch.from_numpy(np.repeat(v, g, axis=0))[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)[0]
    n = q.shape[1]
    s = torch.einsum("hnd,hmd->hnm", qt[0], kt[0]) * scale
    causal = torch.ones(n, n, dtype=torch.bool).tril()
    lse = torch.logsumexp(s.masked_fill(~causal, float("-inf")), dim=-1)
    return o.numpy(), lse.numpy()


@pytest.mark.parametrize("n,B,heads,kv", [(192, 64, 2, 1), (100, 32, 2, 2), (256, 128, 4, 2)])
def test_all_ones_layout_is_dense_causal(n, B, heads, kv):
    d = 32
    q, k, v = _rand(heads, kv, n, d)
    scale = 1 / math.sqrt(d)
    sets = _all_ones(n, B)
    o_ref, lse_ref = _sdpa_causal(q, k, v, scale)
    for fn in (A.forward_dense, A.forward_sparse):
        o, lse = fn(q, k, v, sets, B, scale)
        np.testing.assert_allclose(o, o_ref, atol=1e-12, rtol=0)
        np.testing.assert_allclose(lse, lse_ref, atol=1e-12, rtol=0)


def test_block_diagonal_with_one_chunk_is_causal():
    n = d = 64
    q, k, v = _rand(3, 3, n, d, seed=4)
    scale = 0.3
    sets = L.kept_sets(L.BAND_GLOBAL, n, n, 1, window=0, global_first=0)
    o_ref, lse_ref = _sdpa_causal(q, k, v, scale)
    o, lse = A.forward_dense(q, k, v, sets, n, scale)
    np.testing.assert_allclose(o, o_ref, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12, rtol=0)


def test_block_diagonal_is_per_chunk_causal():
    """BSBR within-chunk term: every chunk is an independent causal problem."""
    n, B, d = 256, 64, 16
    q, k, v = _rand(2, 2, n, d, seed=7)
    scale = 1 / math.sqrt(d)
    sets = L.kept_sets(L.BAND_GLOBAL, n, B, 1, window=0, global_first=0)
    o, lse = A.forward_sparse(q, k, v, sets, B, scale)
    for c in range(n // B):
        sl = slice(c * B, (c + 1) * B)
        o_ref, lse_ref = _sdpa_causal(q[:, sl], k[:, sl], v[:, sl], scale)
        np.testing.assert_allclose(o[:, sl], o_ref, atol=1e-12, rtol=0)
        np.testing.assert_allclose(lse[:, sl], lse_ref, atol=1e-12, rtol=0)


def test_closed_forms():
    n, B, d = 96, 16, 8
    sets = L.kept_sets(L.DYADIC, n, B, 1, window=2, global_first=1)
    q, k, v = _rand(1, 1, n, d, seed=11)
    scale = 0.25
    o, lse = A.forward_dense(q, k, v, sets, B, scale)
    # token 0 sees only itself
    np.testing.assert_array_equal(o[0, 0], v[0, 0])
    assert lse[0, 0] == pytest.approx(scale * float(q[0, 0] @ k[0, 0]), abs=1e-14)
    # Q = 0: uniform weights over the allowed keys
    oz, lz = A.forward_dense(np.zeros_like(q), k, v, sets, B, scale)
    for t in range(n):
        i = t // B
        allowed = [u for j in sorted(sets[0][i]) for u in range(j * B, (j + 1) * B) if j < i or u <= t]
        np.testing.assert_allclose(oz[0, t], v[0, allowed].mean(axis=0), atol=1e-13)
        assert lz[0, t] == pytest.approx(math.log(len(allowed)), abs=1e-13)
    # constant V gives that constant back
    oc, _ = A.forward_sparse(q, k, np.full_like(v, 0.75), sets, B, scale)
    np.testing.assert_allclose(oc, 0.75, atol=1e-14)


def test_rows_sum_to_one_and_lse_consistent():
    n, B, d = 80, 16, 8
    sets = L.kept_sets(L.RANDOM, n, B, 2, density=0.4, seed=3)
    q, k, v = _rand(2, 1, n, d, seed=2)
    scale = 1 / math.sqrt(d)
    o, lse, probs = A.forward_dense(q, k, v, sets, B, scale, return_probs=True)
    for f in range(2):
        np.testing.assert_allclose(probs[f].sum(axis=1), 1.0, atol=1e-12)
        s = scale * q[f] @ k[0].T
        mask = A.token_mask(sets[f % 2], n, B)
        z = np.where(mask, np.exp(s - lse[f][:, None]), 0.0).sum(axis=1)
        np.testing.assert_allclose(z, 1.0, atol=1e-12)


def test_dropped_blocks_and_future_tokens_do_not_matter():
    n, B, d = 128, 16, 8
    sets = L.kept_sets(L.BAND_GLOBAL, n, B, 1, window=1, global_first=1)
    q, k, v = _rand(1, 1, n, d, seed=9)
    scale = 1 / math.sqrt(d)
    o, lse = A.forward_dense(q, k, v, sets, B, scale)
    # perturb K/V in block 3; only rows of blocks keeping 3 (3 and 4) may change
    k2, v2 = k.copy(), v.copy()
    k2[0, 3 * B:4 * B] += 5.0
    v2[0, 3 * B:4 * B] -= 3.0
    o2, lse2 = A.forward_dense(q, k2, v2, sets, B, scale)
    keep = [i for i in range(n // B) if 3 not in sets[0][i]]
    for i in keep:
        sl = slice(i * B, (i + 1) * B)
        np.testing.assert_array_equal(o2[0, sl], o[0, sl])
        np.testing.assert_array_equal(lse2[0, sl], lse[0, sl])
    assert not np.array_equal(o2[0, 3 * B:5 * B], o[0, 3 * B:5 * B])
    # future tokens: changing K/V at u > t never changes row t
    t = 70
    k3, v3 = k.copy(), v.copy()
    k3[0, t + 1:] = 9.0
    v3[0, t + 1:] = -9.0
    o3, lse3 = A.forward_sparse(q, k3, v3, sets, B, scale)
    o_base, lse_base = A.forward_sparse(q, k, v, sets, B, scale)
    np.testing.assert_array_equal(o3[0, :t + 1], o_base[0, :t + 1])
    np.testing.assert_array_equal(lse3[0, :t + 1], lse_base[0, :t + 1])
    assert not np.array_equal(o3[0, t + 1:], o_base[0, t + 1:])


@pytest.mark.parametrize("kind", [L.BAND_GLOBAL, L.DYADIC, L.RANDOM, L.EXPLICIT])
def test_bruteforce_agrees_on_tiny_inputs(kind):
    n, B, d = 18, 4, 8          # ragged last block (18 = 4*4 + 2)
    heads, kv = 4, 2
    q, k, v = _rand(heads, kv, n, d, seed=kind)
    scale = 1 / math.sqrt(d)
    nb = L.n_blocks(n, B)
    mask = None
    if kind == L.EXPLICIT:
        rng = np.random.default_rng(1)
        mask = [[[int(j <= i and (j == i or rng.random() < 0.5)) for j in range(nb)]
                 for i in range(nb)] for _ in range(2)]
        mask[1][2] = [0] * nb          # an empty row: o = 0, lse = -inf
    sets = L.kept_sets(kind, n, B, 2, window=1, global_first=1, density=0.5, seed=3, mask=mask)
    ob, lb = A.forward_bruteforce(q, k, v, sets, B, scale)
    for fn in (A.forward_dense, A.forward_sparse):
        o, lse = fn(q, k, v, sets, B, scale)
        np.testing.assert_allclose(o, ob, atol=1e-12, rtol=0)
        np.testing.assert_allclose(lse, lb, atol=1e-12, rtol=0)
    if kind == L.EXPLICIT:
        assert np.all(np.isneginf(lb[1, 8:12])) and np.all(ob[1, 8:12] == 0)


@pytest.mark.parametrize("name,n", [("tiny_band_global", None), ("bsbr_block_diagonal", None),
                                    ("band_global_32k", 2048), ("bf1_dyadic_gqa_32k", 2048),
                                    ("static_random_131k", 2048)])
def test_sparse_matches_dense_on_workload_patterns(name, n):
    w = WORKLOADS[name]
    n = n or w.n
    heads = min(w.heads, 4)
    kv = max(1, heads // (w.heads // w.kv_heads))
    q, k, v = _rand(heads, kv, n, w.d, seed=3)
    p = w.pattern
    sets = L.kept_sets(p.kind, n, w.B, min(w.layout_heads, heads), p.window, p.global_first,
                       p.dyadic_kmin, p.density, p.seed)
    scale = 1 / math.sqrt(w.d)
    o, lse = A.forward_dense(q, k, v, sets, w.B, scale)
    o2, lse2 = A.forward_sparse(q, k, v, sets, w.B, scale)
    np.testing.assert_allclose(o2, o, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse2, lse, atol=1e-12, rtol=0)


def test_gqa_mapping_matches_repeated_kv():
    """Query slice f reads K/V slice f // (heads / kv_heads)."""
    n, B, d = 64, 16, 8
    sets = L.kept_sets(L.DYADIC, n, B, 1, window=2, global_first=1)
    q, k, v = _rand(6, 2, n, d, seed=5)
    scale = 0.4
    o, lse = A.forward_sparse(q, k, v, sets, B, scale)
    o_rep, lse_rep = A.forward_dense(q, np.repeat(k, 3, axis=0), np.repeat(v, 3, axis=0), sets, B, scale)
    np.testing.assert_allclose(o, o_rep, atol=1e-13)
    np.testing.assert_allclose(lse, lse_rep, atol=1e-13)
    # a wrong (interleaved) grouping would differ
    o_bad, _ = A.forward_dense(q, np.tile(k, (3, 1, 1)), np.tile(v, (3, 1, 1)), sets, B, scale)
    assert not np.allclose(o, o_bad)


def test_planted_mistakes_fail_a_pin(monkeypatch):
    """A dropped scale or a transposed product in the oracle is caught by the
    library-routine pin."""
    n, B, d = 64, 16, 16
    q, k, v = _rand(1, 1, n, d, seed=1)
    scale = 1 / math.sqrt(d)
    sets = _all_ones(n, B)
    o_ref, _ = _sdpa_causal(q, k, v, scale)
    o_noscale, _ = A.forward_dense(q, k, v, sets, B, 1.0)
    assert not np.allclose(o_noscale, o_ref, atol=1e-6)
    real = A._softmax_rows
    monkeypatch.setattr(A, "_softmax_rows", lambda s: real(s.T.copy()))
    o_bad, _ = A.forward_dense(q, k, v, sets, B, scale)
    assert not np.allclose(o_bad, o_ref, atol=1e-6)
