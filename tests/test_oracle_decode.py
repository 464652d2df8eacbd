"""Pins for the oracle decode step (CPU only).

A decode step is row t of the forward over the first t + 1 tokens, so the
paged-cache restatement is checked against the dense and brute-force forward
restatements (independent code: a token mask over the whole sequence, or pure
Python loops), plus the invariants of the paging itself (any page placement
gives the same result; the table is really read) and closed forms.
"""
import math

import numpy as np
import pytest

from oracle import attention as A
from oracle import decode as D
from oracle import layouts as L
from block_sparse_long_bsa_b200 import inputs


def _seq_inputs(batch, H, hkv, n, d, seed=0):
    q, k, v = inputs.qkv_bits(batch * H, batch * hkv, n, d, seeds=(seed, seed + 1, seed + 2))
    return tuple(inputs.bf16_bits_to_f64(x) for x in (q, k, v))


CASES = [
    # kind, n, B, layout heads, batch, H, H_kv, d, pattern
    (L.DYADIC, 300, 64, 1, 2, 4, 2, 32, dict(window=2, global_first=1, dyadic_kmin=2)),
    (L.BAND_GLOBAL, 200, 64, 1, 1, 2, 1, 16, dict(window=1, global_first=1)),
    (L.RANDOM, 520, 128, 4, 2, 4, 4, 32, dict(density=0.4, seed=5)),
    (L.BAND_GLOBAL, 256, 64, 1, 3, 2, 2, 16, dict(window=0, global_first=0)),
]


@pytest.mark.parametrize("case", CASES)
def test_decode_equals_forward_rows(case):
    kind, n, B, Lh, batch, H, hkv, d, pat = case
    sets = L.kept_sets(kind, n, B, Lh, **pat)
    q, k, v = _seq_inputs(batch, H, hkv, n, d)
    scale = 1.0 / math.sqrt(d)
    o_ref, lse_ref = A.forward_dense(q, k, v, sets, B, scale)
    nb = L.n_blocks(n, B)
    rng = np.random.default_rng(11)
    kc, vc, table = D.pages_from_sequences(k, v, batch, B, rng.permutation(batch * nb))
    for positions in ([0] * batch, [n - 1] * batch, list(rng.integers(0, n, batch)),
                      [min(n - 1, B - 1)] * batch, [min(n - 1, B)] * batch):
        qd = np.stack([q[b * H + h, positions[b]] for b in range(batch) for h in range(H)])
        o, lse = D.decode_step(qd, kc, vc, table, positions, sets, B, scale)
        for b in range(batch):
            for h in range(H):
                f = b * H + h
                t = positions[b]
                assert np.allclose(o[f], o_ref[f, t], rtol=0, atol=1e-12)
                assert abs(lse[f] - lse_ref[f, t]) < 1e-12


def test_decode_equals_bruteforce_tiny():
    n, B, d, batch, H, hkv = 24, 4, 8, 2, 2, 1
    sets = L.kept_sets(L.DYADIC, n, B, 1, window=1, global_first=1, dyadic_kmin=2)
    q, k, v = _seq_inputs(batch, H, hkv, n, d, seed=3)
    scale = 0.4
    o_ref, lse_ref = A.forward_bruteforce(q, k, v, sets, B, scale)
    kc, vc, table = D.pages_from_sequences(k, v, batch, B, np.arange(batch * L.n_blocks(n, B)))
    for t in range(n):
        qd = np.stack([q[f, t] for f in range(batch * H)])
        o, lse = D.decode_step(qd, kc, vc, table, [t] * batch, sets, B, scale)
        assert np.allclose(o, o_ref[:, t], atol=1e-12)
        assert np.allclose(lse, lse_ref[:, t], atol=1e-12)


def test_page_placement_does_not_matter_and_the_table_is_read():
    n, B, d, batch, H, hkv = 256, 64, 16, 2, 2, 2
    sets = L.kept_sets(L.BAND_GLOBAL, n, B, 1, window=2, global_first=1)
    q, k, v = _seq_inputs(batch, H, hkv, n, d, seed=7)
    nb = L.n_blocks(n, B)
    pos = [n - 1, 150]
    qd = np.stack([q[b * H + h, pos[b]] for b in range(batch) for h in range(H)])
    kc0, vc0, t0 = D.pages_from_sequences(k, v, batch, B, np.arange(batch * nb))
    kc1, vc1, t1 = D.pages_from_sequences(k, v, batch, B, np.random.default_rng(1).permutation(batch * nb))
    a = D.decode_step(qd, kc0, vc0, t0, pos, sets, B, 0.25)
    b = D.decode_step(qd, kc1, vc1, t1, pos, sets, B, 0.25)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    # planted mistake: sequence 1 (token 150, block 2, keeping blocks 0-2)
    # has a kept block's table entry swapped with block 3's, data unmoved
    bad = t1.copy()
    bad[1, 1], bad[1, 3] = bad[1, 3], bad[1, 1]
    c = D.decode_step(qd, kc1, vc1, bad, pos, sets, B, 0.25)
    assert np.array_equal(c[0][:H], a[0][:H])
    assert not np.allclose(c[0][H:], a[0][H:])


def test_closed_forms():
    n, B, d, batch, H, hkv = 130, 64, 8, 1, 2, 1
    sets = L.kept_sets(L.DYADIC, n, B, 1, window=2, global_first=1, dyadic_kmin=2)
    q, k, v = _seq_inputs(batch, H, hkv, n, d, seed=9)
    kc, vc, table = D.pages_from_sequences(k, v, batch, B, np.arange(L.n_blocks(n, B)))
    scale = 1.0 / math.sqrt(d)
    # token 0 sees only itself
    o, lse = D.decode_step(q[:, 0], kc, vc, table, [0], sets, B, scale)
    assert np.allclose(o, np.repeat(v[:1, 0], H, axis=0), atol=1e-15)
    assert np.allclose(lse, scale * (q[:, 0] @ k[0, 0]), atol=1e-12)
    # q = 0: uniform weights over the allowed keys
    t = 129
    o, lse = D.decode_step(np.zeros((H, d)), kc, vc, table, [t], sets, B, scale)
    allowed = [u for u in range(t + 1) if (u // B) in sets[0][t // B]]
    assert np.allclose(o[0], v[0, allowed].mean(axis=0), atol=1e-12)
    assert abs(lse[0] - math.log(len(allowed))) < 1e-12


def test_empty_row_gives_zero_and_minus_inf():
    n, B, d = 128, 64, 8
    mask = np.zeros((1, 2, 2), dtype=np.uint8)
    mask[0, 0, 0] = 1                           # block 1 keeps nothing
    sets = L.kept_sets(L.EXPLICIT, n, B, 1, mask=mask)
    q, k, v = _seq_inputs(1, 1, 1, n, d)
    kc, vc, table = D.pages_from_sequences(k, v, 1, B, np.arange(2))
    o, lse = D.decode_step(q[:, 100], kc, vc, table, [100], sets, B, 1.0)
    assert np.all(o == 0) and lse[0] == -np.inf
