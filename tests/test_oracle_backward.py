"""Pins for the oracle backward (CPU only).

* Directional finite differences of the forward restatement (a different
  code path: the loss sum(o * dO) is re-evaluated at perturbed inputs).
* torch's autograd of scaled_dot_product_attention (a library routine) on the
  layouts that reduce to dense causal attention, with grouped-query heads.
* Keys that no query reads get exactly zero gradient; a planted sign error in
  the Jacobian is caught by the finite differences.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import backward as BW
from oracle import layouts as L
from block_sparse_long_bsa_b200 import inputs


def _rand(heads, kv_heads, n, d, seed=0):
    q, k, v = inputs.qkv_bits(heads, kv_heads, n, d, seeds=(seed, seed + 1, seed + 2))
    return tuple(inputs.bf16_bits_to_f64(x) for x in (q, k, v))


def _loss(q, k, v, do, sets, B, scale):
    o, _ = A.forward_dense(q, k, v, sets, B, scale)
    return float(np.sum(o * do))


PATTERNS = [
    (L.DYADIC, 40, 4, 1, dict(window=1, global_first=1, dyadic_kmin=2)),
    (L.BAND_GLOBAL, 36, 8, 1, dict(window=1, global_first=1)),
    (L.RANDOM, 48, 8, 2, dict(density=0.5, seed=3)),
]


@pytest.mark.parametrize("pat", PATTERNS)
def test_directional_finite_differences(pat):
    kind, n, B, Lh, kw = pat
    heads, kv, d = 4, 2, 8
    sets = L.kept_sets(kind, n, B, Lh, **kw)
    q, k, v = _rand(heads, kv, n, d, seed=5)
    rng = np.random.default_rng(1)
    do = rng.standard_normal(q.shape)
    scale = 0.37
    dq, dk, dv = BW.backward_dense(q, k, v, do, sets, B, scale)
    eps = 1e-5
    for which, grad in (("q", dq), ("k", dk), ("v", dv)):
        for _ in range(3):
            e = rng.standard_normal(grad.shape)
            args = {"q": q, "k": k, "v": v}
            plus = dict(args); plus[which] = args[which] + eps * e
            minus = dict(args); minus[which] = args[which] - eps * e
            fd = (_loss(plus["q"], plus["k"], plus["v"], do, sets, B, scale)
                  - _loss(minus["q"], minus["k"], minus["v"], do, sets, B, scale)) / (2 * eps)
            an = float(np.sum(grad * e))
            assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (which, fd, an)


def test_matches_torch_autograd_dense_causal_gqa():
    n, B, d, heads, kv = 64, 8, 16, 4, 2
    nb = L.n_blocks(n, B)
    sets = [[set(range(i + 1)) for i in range(nb)]]          # every earlier block kept
    q, k, v = _rand(heads, kv, n, d, seed=9)
    do = np.random.default_rng(2).standard_normal(q.shape)
    scale = 1.0 / math.sqrt(d)
    dq, dk, dv = BW.backward_dense(q, k, v, do, sets, B, scale)
    g = heads // kv
    qt = torch.from_numpy(q).requires_grad_()
    kt = torch.from_numpy(k).requires_grad_()
    vt = torch.from_numpy(v).requires_grad_()
    o = torch.nn.functional.scaled_dot_product_attention(
        qt[None], kt.repeat_interleave(g, 0)[None], vt.repeat_interleave(g, 0)[None],
        is_causal=True, scale=scale)[0]
    o.backward(torch.from_numpy(do))
    assert np.allclose(dq, qt.grad.numpy(), atol=1e-12)
    assert np.allclose(dk, kt.grad.numpy(), atol=1e-12)
    assert np.allclose(dv, vt.grad.numpy(), atol=1e-12)


def test_unread_keys_get_zero_gradient():
    # block-diagonal: keys of block j are read only by queries of block j;
    # with the explicit mask below block 2's keys are read by nobody
    n, B, d = 48, 8, 8
    nb = L.n_blocks(n, B)
    mask = np.zeros((1, nb, nb), dtype=np.uint8)
    for i in range(nb):
        mask[0, i, i] = 1 if i != 2 else 0
        mask[0, i, 0] = 1
    mask[0, 2, 0] = 1
    sets = L.kept_sets(L.EXPLICIT, n, B, 1, mask=mask)
    q, k, v = _rand(1, 1, n, d, seed=4)
    do = np.random.default_rng(3).standard_normal(q.shape)
    dq, dk, dv = BW.backward_dense(q, k, v, do, sets, B, 0.5)
    assert np.all(dk[0, 2 * B:3 * B] == 0) and np.all(dv[0, 2 * B:3 * B] == 0)
    assert np.any(dk[0, 3 * B:4 * B] != 0)


def test_planted_sign_error_is_caught():
    n, B, d, heads, kv = 32, 8, 8, 2, 1
    sets = L.kept_sets(L.DYADIC, n, B, 1, window=1, global_first=1, dyadic_kmin=2)
    q, k, v = _rand(heads, kv, n, d, seed=6)
    do = np.random.default_rng(4).standard_normal(q.shape)
    dq, dk, dv = BW.backward_dense(q, k, v, do, sets, B, 0.3)
    e = np.random.default_rng(5).standard_normal(q.shape)
    eps = 1e-5
    fd = (_loss(q + eps * e, k, v, do, sets, B, 0.3) - _loss(q - eps * e, k, v, do, sets, B, 0.3)) / (2 * eps)
    assert abs(fd - np.sum(dq * e)) < 1e-7
    assert abs(fd - np.sum(-dq * e)) > 1e-3          # the flipped Jacobian fails the same check


@pytest.mark.parametrize("pat", PATTERNS)
def test_block_restatements_match_dense(pat):
    kind, n, B, Lh, kw = pat
    heads, kv, d = 4, 2, 8
    sets = L.kept_sets(kind, n, B, Lh, **kw)
    q, k, v = _rand(heads, kv, n, d, seed=8)
    do = np.random.default_rng(6).standard_normal(q.shape)
    dq, dk, dv = BW.backward_dense(q, k, v, do, sets, B, 0.41)
    nb = L.n_blocks(n, B)
    for f in range(heads):
        for i in range(nb):
            rows = BW.backward_block_dq(q, k, v, do, sets, B, 0.41, f, i)
            assert np.allclose(rows, dq[f, i * B:i * B + rows.shape[0]], atol=1e-12)
    for kh in range(kv):
        for j in range(nb):
            bk, bv = BW.backward_block_dkv(q, k, v, do, sets, B, 0.41, kh, j)
            assert np.allclose(bk, dk[kh, j * B:j * B + bk.shape[0]], atol=1e-12)
            assert np.allclose(bv, dv[kh, j * B:j * B + bv.shape[0]], atol=1e-12)
