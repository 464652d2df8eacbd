"""GPU parity of bsa_backward (through the C ABI) against the fp64 oracle
backward, on the forward's own outputs (o, lse), every pattern family,
grouped-query heads with and without packing, per-head layouts, ragged
sequence ends, unread key blocks and empty rows, and sampled rows of the
full 32K dyadic geometry.

Tolerance.  The kernels form S and dP exactly in fp32 from the bf16 inputs
and rebuild P in fp32 from the forward's lse; the products that produce the
gradients take P and dS = P (dP - D) rounded to bf16 (relative error at most
2^-8 per term, bf16's unit roundoff), and D uses the forward's bf16 o.  Each
gradient element is a sum of such terms, so its error is at most about 2^-8
of the sum of the terms' magnitudes; with independent rounding the normwise
error is far smaller (about 1.7e-3 is measured).  The test asks for a normwise relative error
||g - g_ref|| / ||g_ref|| <= 1e-2 and max |g - g_ref| <= 2e-2 max |g_ref|
on each of dq, dk, dv.
"""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import block_sparse_long_bsa_b200 as bsa
from block_sparse_long_bsa_b200 import inputs
from oracle import backward as BW
from oracle import layouts as OL

from gpu_common import to_device_bf16

pytestmark = pytest.mark.gpu

REL_FRO_TOL = 1e-2
REL_MAX_TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    bsa.load_library()


def grad_errors(g, ref):
    g = np.asarray(g, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = np.abs(g - ref)
    nref = float(np.linalg.norm(ref))
    fro = float(np.linalg.norm(g - ref)) / nref if nref > 0 else float(np.linalg.norm(g - ref))
    big = float(np.abs(ref).max()) if ref.size else 0.0
    return fro, float(diff.max()) if diff.size else 0.0, big


def assert_grad_close(g, ref, what):
    fro, mx, big = grad_errors(g, ref)
    print(f"{what}: rel fro {fro:.3e}  max {mx:.3e}  (max |ref| {big:.3e})")
    assert fro <= REL_FRO_TOL, f"{what}: normwise relative error {fro:.3e}"
    assert mx <= REL_MAX_TOL * max(big, 1e-6), f"{what}: max error {mx:.3e} vs max |ref| {big:.3e}"


def _run(kind, n, B, Lh, heads, kv, d, pat, seed=0, mask=None):
    dev = torch.cuda.current_device()
    extra = dict(pat)
    if mask is not None:
        extra["mask"] = mask
    lay = bsa.Layout(kind, n, B, Lh, dev, **extra)
    sets = OL.kept_sets(kind, n, B, Lh, **extra)
    qb, kb, vb = inputs.qkv_bits(heads, kv, n, d, seeds=(seed, seed + 1, seed + 2))
    dob = inputs.normal_bf16_bits((heads, n, d), seed + 3)
    q, k, v, do = (to_device_bf16(x) for x in (qb, kb, vb, dob))
    scale = 1.0 / math.sqrt(d)
    o, lse = bsa.attention(q, k, v, lay, scale=scale)
    dq, dk, dv = bsa.attention_backward(q, k, v, o, lse, do, lay, scale=scale)
    torch.cuda.synchronize()
    bsa.bsa_get_status(lay.handle)
    host = tuple(inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb, dob))
    return lay, sets, host, (q, k, v, o, lse, do), (dq.cpu().numpy(), dk.cpu().numpy(), dv.cpu().numpy()), scale


CASES = [
    # kind, n, B, layout heads, heads, kv heads, d, pattern
    (OL.DYADIC, 1000, 64, 1, 4, 2, 128, dict(window=2, global_first=1, dyadic_kmin=2)),      # packed pairs, ragged
    (OL.BAND_GLOBAL, 777, 128, 1, 2, 2, 128, dict(window=1, global_first=1)),                # B = 128, ragged
    (OL.RANDOM, 1024, 128, 2, 4, 1, 64, dict(density=0.4, seed=5)),                          # per-head layouts, d = 64
    (OL.BAND_GLOBAL, 640, 64, 1, 3, 1, 64, dict(window=1, global_first=1)),                  # odd group: no packing
    (OL.RANDOM, 1536, 64, 2, 4, 2, 128, dict(density=0.5, seed=9)),                          # B = 64, per-head layouts
    (OL.DYADIC, 2500, 128, 1, 2, 1, 64, dict(window=2, global_first=1, dyadic_kmin=2)),      # B = 128, d = 64
    (OL.BAND_GLOBAL, 4096, 64, 1, 2, 1, 128, dict(window=0, global_first=1)),                # block 0 read by 64 rows
]


@pytest.mark.parametrize("case", CASES)
def test_backward_parity(case):
    kind, n, B, Lh, heads, kv, d, pat = case
    lay, sets, host, dev_t, got, scale = _run(kind, n, B, Lh, heads, kv, d, pat)
    q, k, v, do = host
    ref = BW.backward_dense(q, k, v, do, sets, B, scale)
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        assert_grad_close(g, r, f"{kind} n{n} B{B} d{d} h{heads}/{kv} L{Lh} {name}")
    lay.close()


def test_backward_unread_keys_and_empty_rows():
    # explicit mask: block 2 keeps nothing (its rows are empty, o = 0) and no
    # block keeps block 3, so block 3's keys get exactly zero gradient
    n, B, d = 512, 64, 128
    nb = OL.n_blocks(n, B)
    mask = np.zeros((1, nb, nb), dtype=np.uint8)
    for i in range(nb):
        if i == 2:
            continue
        mask[0, i, 0] = 1
        if i != 3:
            mask[0, i, i] = 1
    lay, sets, host, dev_t, got, scale = _run(OL.EXPLICIT, n, B, 1, 2, 1, d, {}, seed=4, mask=mask)
    dq, dk, dv = got
    assert np.all(dq[:, 2 * B:3 * B] == 0)
    assert np.all(dk[:, 3 * B:4 * B] == 0) and np.all(dv[:, 3 * B:4 * B] == 0)
    ref = BW.backward_dense(*host, sets, B, scale)
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        assert_grad_close(g, r, f"explicit {name}")
    lay.close()


def test_dq_is_deterministic():
    kind, n, B, Lh, heads, kv, d, pat = CASES[0]
    lay, sets, host, dev_t, got, scale = _run(kind, n, B, Lh, heads, kv, d, pat)
    q, k, v, o, lse, do = dev_t
    dq2, dk2, dv2 = bsa.attention_backward(q, k, v, o, lse, do, lay, scale=scale)
    torch.cuda.synchronize()
    assert np.array_equal(dq2.cpu().numpy(), got[0])
    assert np.allclose(dk2.cpu().numpy(), got[1], rtol=0, atol=1e-5 * max(1.0, float(np.abs(got[1]).max())))
    lay.close()


def test_backward_full_32k_dyadic_sampled():
    # the headline geometry: 16 query heads on 8 kv heads, n = 32768, B = 64
    n, B, heads, kv, d = 32768, 64, 16, 8, 128
    pat = dict(window=2, global_first=1, dyadic_kmin=2)
    lay, sets, host, dev_t, got, scale = _run(OL.DYADIC, n, B, 1, heads, kv, d, pat, seed=11)
    q, k, v, do = host
    dq, dk, dv = got
    nb = OL.n_blocks(n, B)
    for f, i in ((0, 0), (3, nb - 1), (8, 257), (15, 100)):
        ref = BW.backward_block_dq(q, k, v, do, sets, B, scale, f, i)
        assert_grad_close(dq[f, i * B:(i + 1) * B], ref, f"32K dq head {f} block {i}")
    # block 0 is read by every query block (many column segments, summed
    # across CTAs); the others by a handful
    for kh, j in ((0, 0), (5, nb - 1), (2, 300), (7, 64)):
        rk, rv = BW.backward_block_dkv(q, k, v, do, sets, B, scale, kh, j)
        assert_grad_close(dk[kh, j * B:(j + 1) * B], rk, f"32K dk kv head {kh} block {j}")
        assert_grad_close(dv[kh, j * B:(j + 1) * B], rv, f"32K dv kv head {kh} block {j}")
    lay.close()


def test_backward_invalid_arguments_launch_nothing():
    n, B, heads, kv, d = 256, 64, 2, 1, 64
    dev = torch.cuda.current_device()
    lay = bsa.Layout(OL.BAND_GLOBAL, n, B, 1, dev, window=1, global_first=1)
    bf = dict(dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((heads, n, d), **bf)
    k = torch.zeros((kv, n, d), **bf)
    o = torch.zeros((heads, n, d), **bf)
    lse = torch.zeros((heads, n), dtype=torch.float32, device="cuda")
    dq = torch.full((heads, n, d), 7.0, dtype=torch.float32, device="cuda")
    dk = torch.full((kv, n, d), 7.0, dtype=torch.float32, device="cuda")
    dv = torch.full((kv, n, d), 7.0, dtype=torch.float32, device="cuda")
    ws = torch.full((heads, n), 7.0, dtype=torch.float32, device="cuda")
    calls = [dict(B=128), dict(n=n - 1), dict(d=96), dict(kv_heads=3), dict(heads=0), dict(scale=-1.0),
             dict(scale=float("nan")), dict(dq=0), dict(workspace=0), dict(dk=dk.data_ptr() + 4)]
    for bad in calls:
        args = dict(B=B, n=n, heads=heads, kv_heads=kv, d=d, scale=0.1, dq=dq, dk=dk, workspace=ws)
        args.update(bad)
        with pytest.raises(bsa.BsaError):
            bsa.bsa_backward(q, k, k, o, lse, q, lay.handle, args["B"], args["n"], args["heads"],
                             args["kv_heads"], args["d"], args["scale"], args["dq"], args["dk"], dv,
                             args["workspace"])
    torch.cuda.synchronize()
    assert torch.all(dq == 7.0) and torch.all(dk == 7.0) and torch.all(dv == 7.0) and torch.all(ws == 7.0)
    lay.close()
