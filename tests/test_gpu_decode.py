"""GPU parity of bsa_decode (through the C ABI) against the fp64 oracle decode
step, on shuffled page tables, every pattern family, packed grouped-query
heads, ragged sequence ends, block-boundary positions and the full 32K
dyadic geometry.  Tolerances as for the forward: max |d| <= 1e-2 and
mean |d| <= 1e-3 on o and lse.
"""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import block_sparse_long_bsa_b200 as bsa
from block_sparse_long_bsa_b200 import inputs
from oracle import decode as D
from oracle import layouts as OL

from gpu_common import assert_close, to_device_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    bsa.load_library()


def _setup(kind, n, B, Lh, batch, H, hkv, d, pat, seed=0):
    dev = torch.cuda.current_device()
    lay = bsa.Layout(kind, n, B, Lh, dev, **pat)
    sets = OL.kept_sets(kind, n, B, Lh, **pat)
    qb, kb, vb = inputs.qkv_bits(batch * H, batch * hkv, n, d, seeds=(seed, seed + 1, seed + 2))
    nb = OL.n_blocks(n, B)
    order = np.random.default_rng(seed + 100).permutation(batch * nb)
    kcb, vcb, table = D.pages_from_sequences(kb, vb, batch, B, order)
    dev_t = dict(kc=to_device_bf16(kcb), vc=to_device_bf16(vcb),
                 table=torch.from_numpy(table).to("cuda"))
    host = dict(q=qb, kc=inputs.bf16_bits_to_f64(kcb), vc=inputs.bf16_bits_to_f64(vcb), table=table)
    return lay, sets, dev_t, host


def _step(lay, sets, dev_t, host, batch, H, d, B, positions, scale):
    qrows = np.stack([host["q"][b * H + h, positions[b]] for b in range(batch) for h in range(H)])
    q = to_device_bf16(qrows)
    pos = torch.tensor(positions, dtype=torch.int32, device="cuda")
    o, lse = bsa.decode(q, dev_t["kc"], dev_t["vc"], dev_t["table"], pos, lay, batch, scale=scale)
    torch.cuda.synchronize()
    o_ref, lse_ref = D.decode_step(inputs.bf16_bits_to_f64(qrows), host["kc"], host["vc"], host["table"],
                                   positions, sets, B, scale)
    return o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref


CASES = [
    (OL.DYADIC, 4096, 64, 1, 2, 4, 2, 128, dict(window=2, global_first=1, dyadic_kmin=2)),
    (OL.RANDOM, 4096, 128, 4, 2, 4, 4, 128, dict(density=0.3, seed=4)),
    (OL.BAND_GLOBAL, 1000, 64, 1, 3, 2, 1, 64, dict(window=2, global_first=1)),
    (OL.BAND_GLOBAL, 1500, 128, 1, 2, 2, 2, 64, dict(window=1, global_first=1)),
]


@pytest.mark.parametrize("case", CASES)
def test_decode_parity(case):
    kind, n, B, Lh, batch, H, hkv, d, pat = case
    lay, sets, dev_t, host = _setup(kind, n, B, Lh, batch, H, hkv, d, pat)
    scale = 1.0 / math.sqrt(d)
    rng = np.random.default_rng(5)
    for positions in ([0] * batch, [n - 1] * batch, [B - 1] * batch, [B] * batch,
                      [int(x) for x in rng.integers(0, n, batch)]):
        o, lse, o_ref, lse_ref = _step(lay, sets, dev_t, host, batch, H, d, B, positions, scale)
        assert_close(o, lse, o_ref, lse_ref, f"{kind} B{B} d{d} positions {positions}")
    bsa.bsa_get_status(lay.handle)
    lay.close()


def test_decode_full_32k_dyadic():
    n, B, batch, H, hkv, d = 32768, 64, 4, 16, 8, 128
    lay, sets, dev_t, host = _setup(OL.DYADIC, n, B, 1, batch, H, hkv, d,
                                    dict(window=2, global_first=1, dyadic_kmin=2), seed=3)
    o, lse, o_ref, lse_ref = _step(lay, sets, dev_t, host, batch, H, d, B, [n - 1, 20000, 4097, 65],
                                   1.0 / math.sqrt(d))
    assert_close(o, lse, o_ref, lse_ref, "decode 32K dyadic")
    bsa.bsa_get_status(lay.handle)
    lay.close()


def test_decode_cluster_shapes():
    """The launch shapes the host picks at the ends of its range: a one-block
    route (BSBR's block-diagonal layout: four tasks a row, one CTA per
    cluster) and so many query groups (25 sequences x 8 key/value heads) that
    the clusters shrink to fit the GPU at once (to two CTAs on a 148-SM
    B200, the shape of a batch-32 decode of the 32K route)."""
    for kind, n, B, batch, H, hkv, d, pat in (
            (OL.BAND_GLOBAL, 1024, 64, 2, 4, 2, 64, dict(window=0, global_first=0)),
            (OL.DYADIC, 2048, 64, 25, 16, 8, 128, dict(window=2, global_first=1, dyadic_kmin=2))):
        scale = 1.0 / math.sqrt(d)
        lay, sets, dev_t, host = _setup(kind, n, B, 1, batch, H, hkv, d, pat, seed=11)
        rng = np.random.default_rng(12)
        for positions in ([n - 1] * batch, [int(x) for x in rng.integers(0, n, batch)]):
            o, lse, o_ref, lse_ref = _step(lay, sets, dev_t, host, batch, H, d, B, positions, scale)
            assert_close(o, lse, o_ref, lse_ref, f"{kind} n{n} batch {batch}")
        bsa.bsa_get_status(lay.handle)
        lay.close()


def test_decode_long_rows_many_tasks_per_warp():
    """Full causal rows of up to 512 pages: each warp of a cluster takes more
    than 32 tasks of 32 key rows, so its page numbers are fetched in several
    rounds; positions 31 and 32 put the token at the end of a task and at the
    first key of the next one."""
    n, B, batch, H, hkv, d = 32768, 64, 1, 2, 1, 128
    nb = n // B
    lay, sets, dev_t, host = _setup(OL.BAND_GLOBAL, n, B, 1, batch, H, hkv, d,
                                    dict(window=nb, global_first=0), seed=7)
    for positions in ([n - 1], [n // 2 + 5], [31], [32]):
        o, lse, o_ref, lse_ref = _step(lay, sets, dev_t, host, batch, H, d, B, positions, 1.0 / math.sqrt(d))
        assert_close(o, lse, o_ref, lse_ref, f"decode full causal rows, positions {positions}")
    bsa.bsa_get_status(lay.handle)
    lay.close()


def test_decode_refuses_bad_indices_on_device():
    n, B, batch, H, hkv, d = 1024, 64, 2, 2, 2, 64
    lay, sets, dev_t, host = _setup(OL.DYADIC, n, B, 1, batch, H, hkv, d,
                                    dict(window=2, global_first=1, dyadic_kmin=2))
    scale = 1.0 / math.sqrt(d)
    qrows = np.stack([host["q"][f, 500] for f in range(batch * H)])
    q = to_device_bf16(qrows)
    # sequence 0 at a position past the layout's n: its rows are refused
    pos = torch.tensor([n + 5, 500], dtype=torch.int32, device="cuda")
    o, lse = bsa.decode(q, dev_t["kc"], dev_t["vc"], dev_t["table"], pos, lay, batch, scale=scale)
    torch.cuda.synchronize()
    with pytest.raises(bsa.BsaError):
        bsa.bsa_get_status(lay.handle)
    o_ref, lse_ref = D.decode_step(inputs.bf16_bits_to_f64(qrows), host["kc"], host["vc"], host["table"],
                                   [0, 500], sets, B, scale)
    assert torch.all(o[:H] == 0) and torch.all(torch.isneginf(lse[:H]))
    assert_close(o[H:].float().cpu().numpy(), lse[H:].cpu().numpy(), o_ref[H:], lse_ref[H:], "good rows")
    # a page number past the cache: that row is refused, the status reports it
    bad = dev_t["table"].clone()
    bad[1, 500 // B] = 10 ** 6
    pos = torch.tensor([500, 500], dtype=torch.int32, device="cuda")
    o, lse = bsa.decode(q, dev_t["kc"], dev_t["vc"], bad, pos, lay, batch, scale=scale)
    torch.cuda.synchronize()
    with pytest.raises(bsa.BsaError):
        bsa.bsa_get_status(lay.handle)
    assert torch.all(o[H:] == 0) and torch.all(torch.isneginf(lse[H:]))
    assert torch.all(torch.isfinite(lse[:H]))
    bsa.bsa_get_status(lay.handle)          # cleared by the read
    lay.close()


def test_decode_invalid_arguments_launch_nothing():
    n, B, batch, H, hkv, d = 512, 64, 1, 2, 1, 64
    lay, sets, dev_t, host = _setup(OL.BAND_GLOBAL, n, B, 1, batch, H, hkv, d, dict(window=1, global_first=1))
    q = torch.zeros((H, d), dtype=torch.bfloat16, device="cuda")
    o = torch.full((H, d), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((H,), 7.0, dtype=torch.float32, device="cuda")
    pos = torch.zeros((batch,), dtype=torch.int32, device="cuda")
    nb = OL.n_blocks(n, B)
    calls = [
        dict(max_blocks=nb - 1),          # table too narrow for the layout
        dict(d=96),                       # unsupported head dim
        dict(batch=2),                    # heads and kv heads not multiples of the batch
        dict(kv_heads=3),                 # query heads not a multiple of the kv heads
        dict(num_pages=0),
        dict(scale=-1.0),
    ]
    for bad in calls:
        args = dict(max_blocks=nb, heads=H, kv_heads=batch * hkv, batch=batch, d=d, scale=0.1,
                    num_pages=dev_t["kc"].shape[0])
        args.update(bad)
        with pytest.raises(bsa.BsaError):
            bsa.bsa_decode(q, dev_t["kc"], dev_t["vc"], dev_t["table"], args["max_blocks"],
                           args["num_pages"], pos, lay.handle, args["batch"], args["heads"],
                           args["kv_heads"], args["d"], args["scale"], o, lse)
    torch.cuda.synchronize()
    assert torch.all(o == 7.0) and torch.all(lse == 7.0)
    lay.close()
