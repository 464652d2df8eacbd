"""bsa_forward_host (through the C ABI): the forward from and to host memory,
cut into runs of key/value heads whose copies overlap the other runs'
compute, against bsa_forward on the same inputs.  Every (head, query block)
tile is computed by the same kernel code whichever launch takes it, so o and
lse must agree bit for bit; layouts with several layout heads check that the
runs start on layout head 0."""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import block_sparse_long_bsa_b200 as bsa
from block_sparse_long_bsa_b200 import inputs
from oracle import layouts as OL

from gpu_common import to_device_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    bsa.load_library()


def _pinned(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).pin_memory()


CASES = [
    # kind, n, B, layout heads, heads, kv heads, d, pattern, groups
    (OL.DYADIC, 2048, 64, 1, 8, 4, 128, dict(window=2, global_first=1, dyadic_kmin=2), 3),
    (OL.RANDOM, 2048, 128, 2, 8, 8, 64, dict(density=0.3, seed=4), 3),
    (OL.BAND_GLOBAL, 1000, 64, 1, 4, 2, 64, dict(window=1, global_first=1), 8),
]


@pytest.mark.parametrize("case", CASES)
def test_forward_host_matches_device_forward(case):
    kind, n, B, L, heads, kv, d, pat, groups = case
    scale = 1.0 / math.sqrt(d)
    lay = bsa.Layout(kind, n, B, L, torch.cuda.current_device(), **pat)
    qb, kb, vb = inputs.qkv_bits(heads, kv, n, d, seeds=(51, 52, 53))
    hq, hk, hv = _pinned(qb), _pinned(kb), _pinned(vb)
    q = torch.empty(hq.shape, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(hk.shape, dtype=torch.bfloat16, device="cuda")
    v = torch.empty(hv.shape, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((heads, n), dtype=torch.float32, device="cuda")
    ho = torch.empty(hq.shape, dtype=torch.bfloat16).pin_memory()
    hl = torch.empty((heads, n), dtype=torch.float32).pin_memory()
    bsa.bsa_forward_host(hq, hk, hv, lay.handle, B, n, heads, kv, d, scale, q, k, v, o, lse, ho, hl, groups)
    torch.cuda.current_stream().synchronize()
    bsa.bsa_get_status(lay.handle)
    o_ref, lse_ref = bsa.attention(to_device_bf16(qb), to_device_bf16(kb), to_device_bf16(vb), lay, scale)
    torch.cuda.synchronize()
    assert torch.equal(ho, o_ref.cpu()), "o differs from the device forward"
    assert torch.equal(hl, lse_ref.cpu()), "lse differs from the device forward"
    lay.close()


def test_forward_host_invalid_arguments_launch_nothing():
    n, B, heads, kv, d = 512, 64, 2, 1, 64
    lay = bsa.Layout(OL.BAND_GLOBAL, n, B, 1, torch.cuda.current_device(), window=1, global_first=1)
    hq = torch.zeros((heads, n, d), dtype=torch.bfloat16).pin_memory()
    hk = torch.zeros((kv, n, d), dtype=torch.bfloat16).pin_memory()
    q = torch.empty(hq.shape, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(hk.shape, dtype=torch.bfloat16, device="cuda")
    v = torch.empty(hk.shape, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((heads, n), dtype=torch.float32, device="cuda")
    ho = torch.full(hq.shape, 7.0, dtype=torch.bfloat16).pin_memory()
    hl = torch.full((heads, n), 7.0, dtype=torch.float32).pin_memory()
    for bad in (dict(v_host=None), dict(groups=0), dict(d=96)):
        args = dict(v_host=hk, groups=2, d=d)
        args.update(bad)
        with pytest.raises(bsa.BsaError):
            bsa.bsa_forward_host(hq, hk, args["v_host"], lay.handle, B, n, heads, kv, args["d"], 0.125,
                                 q, k, v, o, lse, ho, hl, args["groups"])
    torch.cuda.synchronize()
    assert torch.all(ho == 7.0) and torch.all(hl == 7.0)
    lay.close()
