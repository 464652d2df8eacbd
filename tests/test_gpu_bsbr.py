"""GPU parity of BSBR attention (bsa_forward on the block-diagonal layout,
then bsa_bsbr_retrieval through the C ABI) against the fp64 oracle: the
retrieval term alone and the summed output, on the BSBR workload (batch 2 x
8 heads, n = 4096, d = 64, B = 128), both block sizes, both head dims,
grouped-query heads and ragged ends.

Tolerance.  The retrieval is computed with fp32 sums, exact bf16 x bf16
products and a state split into bf16 hi + lo parts (relative error about
2^-16), and the result is rounded to bf16 once.  That rounding moves a value
by at most half the gap between bf16 neighbours at the rounded value
(``bf16_half_ulp``, a property of round-to-nearest, pinned on the CPU), so
each bound is that allowance plus an arithmetic budget, and only the
arithmetic can use up the budget, never the luck of where a value falls
between two bf16 numbers:
  retrieval term alone:  |o - o_ref| <= half_ulp(o) + 1e-4 max |ref|
  summed output:         |o - o_ref| <= half_ulp(o) + 1.5e-2
(the within-chunk term's own 1e-2 bound, its rounding to bf16 before the
add, and the retrieval's arithmetic).  Both are tighter than the relative
2^-8 |ref| allowance they replace, which equals half_ulp only at the bottom
of each binade.  Each test prints the worst share of its bound and the
worst share of the arithmetic budget left after the rounding allowance.
"""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import block_sparse_long_bsa_b200 as bsa
from block_sparse_long_bsa_b200 import inputs
from oracle import attention as OA
from oracle import bsbr as BS
from oracle import layouts as OL

from gpu_common import bf16_half_ulp, to_device_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    bsa.load_library()


def _inputs(heads, kv, n, d, seed):
    qb, kb, vb = inputs.qkv_bits(heads, kv, n, d, seeds=(seed, seed + 1, seed + 2))
    return (qb, kb, vb), tuple(to_device_bf16(x) for x in (qb, kb, vb)), \
        tuple(inputs.bf16_bits_to_f64(x) for x in (qb, kb, vb))


def _layout(n, B):
    return bsa.Layout(OL.BAND_GLOBAL, n, B, 1, torch.cuda.current_device(), window=0, global_first=0)


def _workspace(n, B, kv, d):
    need = bsa.bsa_bsbr_workspace_bytes(n, B, kv, d)
    ws = torch.empty(((need + 15) // 16) * 4, dtype=torch.float32, device="cuda")
    return ws, ws.numel() * 4


CASES = [
    # heads, kv heads, n, d, B
    (16, 16, 4096, 64, 128),      # the BSBR workload: batch 2 x 8 heads
    (4, 2, 1000, 128, 64),
    (2, 1, 777, 128, 128),
    (3, 3, 256, 64, 64),
    (2, 2, 64 * 40 + 1, 64, 64),  # a one-token last chunk
]


@pytest.mark.parametrize("case", CASES)
def test_retrieval_term_alone(case):
    heads, kv, n, d, B = case
    _, (q, k, v), (qh, kh, vh) = _inputs(heads, kv, n, d, seed=21)
    lay = _layout(n, B)
    scale = 1.0 / math.sqrt(d)
    o = torch.zeros((heads, n, d), dtype=torch.bfloat16, device="cuda")
    ws, nbytes = _workspace(n, B, kv, d)
    bsa.bsa_bsbr_retrieval(q, k, v, lay.handle, B, n, heads, kv, d, scale, o, ws, nbytes)
    torch.cuda.synchronize()
    bsa.bsa_get_status(lay.handle)
    ref = BS.retrieval(qh, kh, vh, B, scale)
    got = o.float().cpu().numpy()
    assert np.all(got[:, :B] == 0)
    err = np.abs(got - ref)
    budget = 1e-4 * np.abs(ref).max()
    bound = bf16_half_ulp(got) + budget
    print(f"retrieval h{heads}/{kv} n{n} d{d} B{B}: max {err.max():.3e} (max |ref| {np.abs(ref).max():.2f}), "
          f"worst share of bound {(err / bound).max():.3f}, "
          f"of arithmetic budget {((err - bf16_half_ulp(got)) / budget).max():.3f}")
    assert np.all(err <= bound)
    lay.close()


@pytest.mark.parametrize("case", CASES)
def test_bsbr_output(case):
    heads, kv, n, d, B = case
    _, (q, k, v), (qh, kh, vh) = _inputs(heads, kv, n, d, seed=5)
    lay = _layout(n, B)
    scale = 1.0 / math.sqrt(d)
    o, lse = bsa.bsbr_attention(q, k, v, lay, scale=scale)
    torch.cuda.synchronize()
    bsa.bsa_get_status(lay.handle)
    o_in, lse_ref = OA.forward_sparse(qh, kh, vh, BS.within_chunk_sets(n, B), B, scale)
    ref = o_in + BS.retrieval(qh, kh, vh, B, scale)
    got = o.float().cpu().numpy()
    err = np.abs(got - ref)
    bound = bf16_half_ulp(got) + 1.5e-2
    print(f"bsbr h{heads}/{kv} n{n} d{d} B{B}: max {err.max():.3e} mean {err.mean():.3e}, "
          f"worst share of bound {(err / bound).max():.3f}, "
          f"of arithmetic budget {((err - bf16_half_ulp(got)) / 1.5e-2).max():.3f}")
    assert np.all(err <= bound)
    assert err.mean() <= 1e-3 + 2.0 ** -9 * np.abs(ref).mean()
    assert np.abs(lse.cpu().numpy() - lse_ref).max() <= 1e-2
    lay.close()


def test_single_chunk_leaves_o_unchanged_and_bad_arguments_launch_nothing():
    heads, kv, n, d, B = 2, 1, 100, 64, 128
    _, (q, k, v), _ = _inputs(heads, kv, n, d, seed=1)
    lay = _layout(n, B)
    o = torch.full((heads, n, d), 3.0, dtype=torch.bfloat16, device="cuda")
    ws, nbytes = _workspace(n, B, kv, d)
    bsa.bsa_bsbr_retrieval(q, k, v, lay.handle, B, n, heads, kv, d, 0.125, o, ws, nbytes)
    torch.cuda.synchronize()
    assert torch.all(o == 3.0)
    lay.close()
    n = 1024
    _, (q, k, v), _ = _inputs(heads, kv, n, d, seed=1)
    lay = _layout(n, B)
    o = torch.full((heads, n, d), 3.0, dtype=torch.bfloat16, device="cuda")
    ws, nbytes = _workspace(n, B, kv, d)
    for bad in (dict(B=64), dict(n=n - 1), dict(d=96), dict(kv_heads=3), dict(scale=0.0),
                dict(nbytes=nbytes - 4), dict(o=o.data_ptr() + 2)):
        a = dict(B=B, n=n, heads=heads, kv_heads=kv, d=d, scale=0.125, nbytes=nbytes, o=o)
        a.update(bad)
        with pytest.raises(bsa.BsaError):
            bsa.bsa_bsbr_retrieval(q, k, v, lay.handle, a["B"], a["n"], a["heads"], a["kv_heads"], a["d"],
                                   a["scale"], a["o"], ws, a["nbytes"])
    torch.cuda.synchronize()
    assert torch.all(o == 3.0)
    lay.close()
