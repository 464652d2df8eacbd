"""GPU parity of bsa_forward (through the C ABI) against the fp64 oracle.

Element-by-element at sizes the oracle finishes in seconds (several tiles,
ragged last blocks, every pattern family, packed and unpacked grouped-query
tiles), and at full size in the launch configuration the benchmark times:
every head and block of the two 32K workloads, and two whole heads plus every
head's longest rows of the 131K workload.  Also: future tokens and dropped
blocks leave o bitwise unchanged, run-to-run bitwise determinism, concurrent
calls on one layout (more in flight than the layout's work counters), invalid
arguments that launch nothing, and the bounded-wait time-out path.
Tolerances: max |d| <= 1e-2 and mean |d| <= 1e-3 on o and lse; layouts
bit-exact (checked on the CPU side).
"""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import block_sparse_long_bsa_b200 as bsa
from block_sparse_long_bsa_b200 import inputs
from block_sparse_long_bsa_b200.workloads import WORKLOADS, Pattern
from oracle import layouts as OL
from oracle import attention as OA

from gpu_common import MAX_ABS_TOL, MEAN_ABS_TOL, assert_close, device_inputs, default_scale

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    bsa.load_library()


def _run(kind, n, B, L, heads, kv, d, scale=None, seeds=(0, 1, 2), **pat):
    scale = scale or default_scale(d)
    lay = bsa.Layout(kind, n, B, L, torch.cuda.current_device(), **pat)
    (qb, kb, vb), (q, k, v) = device_inputs(heads, kv, n, d, seeds)
    o, lse = bsa.attention(q, k, v, lay, scale)
    torch.cuda.synchronize()
    bsa.bsa_get_status(lay.handle)
    sets = OL.kept_sets(kind, n, B, L, **pat)
    return lay, (qb, kb, vb), sets, scale, o.float().cpu().numpy(), lse.cpu().numpy()


def _oracle(qkv_bits, sets, B, scale):
    q, k, v = (inputs.bf16_bits_to_f64(x) for x in qkv_bits)
    return OA.forward_sparse(q, k, v, sets, B, scale)


CASES = [
    # (label, kind, n, B, L, heads, kv, d, pattern)
    ("tiny_band_global", OL.BAND_GLOBAL, 256, 64, 1, 1, 1, 64, dict(window=1, global_first=1)),
    ("bsbr_block_diagonal", OL.BAND_GLOBAL, 4096, 128, 1, 16, 16, 64, dict(window=0, global_first=0)),
    ("band_global_small", OL.BAND_GLOBAL, 2048, 128, 1, 4, 4, 128, dict(window=2, global_first=1)),
    ("band_global_ragged", OL.BAND_GLOBAL, 2048 - 37, 128, 1, 2, 2, 128, dict(window=2, global_first=1)),
    ("dyadic_gqa_small", OL.DYADIC, 4096, 64, 1, 4, 2, 128, dict(window=2, global_first=1, dyadic_kmin=2)),
    ("dyadic_gqa_ragged", OL.DYADIC, 4096 - 5, 64, 1, 4, 2, 128, dict(window=2, global_first=1, dyadic_kmin=2)),
    ("dyadic_mha_unpacked", OL.DYADIC, 2048, 64, 1, 3, 3, 128, dict(window=2, global_first=1, dyadic_kmin=2)),
    ("random_small", OL.RANDOM, 4096, 128, 4, 4, 4, 128, dict(density=0.1, seed=17)),
    ("random_dense_d64", OL.RANDOM, 3000, 128, 2, 4, 2, 64, dict(density=0.5, seed=5)),
    ("random_b64_perhead", OL.RANDOM, 4096, 64, 2, 4, 2, 128, dict(density=0.2, seed=9)),
    ("band_b64_d64_gqa", OL.BAND_GLOBAL, 1024 + 17, 64, 1, 8, 2, 64, dict(window=3, global_first=1)),
    ("all_ones_b128", OL.BAND_GLOBAL, 1024, 128, 1, 2, 1, 128, dict(window=10 ** 6, global_first=1)),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_parity_elementwise(case):
    label, kind, n, B, L, heads, kv, d, pat = case
    lay, bits, sets, scale, o, lse = _run(kind, n, B, L, heads, kv, d, **pat)
    o_ref, lse_ref = _oracle(bits, sets, B, scale)
    assert_close(o, lse, o_ref, lse_ref, label)
    lay.close()


def test_explicit_mask_with_empty_rows():
    n, B, d, L = 1024, 64, 128, 1
    nb = n // B
    rng = np.random.default_rng(3)
    mask = ((rng.random((L, nb, nb)) < 0.4) & np.tri(nb, dtype=bool)[None]).astype(np.uint8)
    mask[0, 3, :] = 0                       # empty row -> o = 0, lse = -inf
    mask[0, 6, 6] = 0                       # a row without its diagonal block
    mask[0, 6, 2] = 1
    lay, bits, sets, scale, o, lse = _run(OL.EXPLICIT, n, B, L, 2, 1, d, mask=mask)
    o_ref, lse_ref = _oracle(bits, sets, B, scale)
    assert np.all(np.isneginf(lse[:, 3 * B:4 * B])) and np.all(o[:, 3 * B:4 * B] == 0)
    assert_close(o, lse, o_ref, lse_ref, "explicit")
    lay.close()


def test_non_default_scale():
    lay, bits, sets, scale, o, lse = _run(OL.DYADIC, 2048, 128, 1, 2, 2, 128, scale=0.05,
                                          window=2, global_first=1, dyadic_kmin=2)
    o_ref, lse_ref = _oracle(bits, sets, 128, 0.05)
    assert_close(o, lse, o_ref, lse_ref, "scale 0.05")
    lay.close()


@pytest.mark.parametrize("kind,n,B,L,heads,kv,d,pat", [
    (OL.BAND_GLOBAL, 2048, 128, 1, 2, 2, 128, dict(window=10 ** 6, global_first=1)),
    (OL.DYADIC, 4096 - 7, 64, 1, 4, 2, 128, dict(window=2, global_first=1, dyadic_kmin=2)),
    (OL.RANDOM, 3072, 128, 2, 2, 2, 64, dict(density=0.4, seed=3)),
])
def test_rescale_path(kind, n, B, L, heads, kv, d, pat):
    """Keys grow in magnitude along the sequence, so each later block's scores
    exceed the running maximum by far more than the rescale threshold and the
    kernel must rescale O (with N(0,1) inputs it essentially never does)."""
    scale = default_scale(d)
    lay = bsa.Layout(kind, n, B, L, torch.cuda.current_device(), **pat)
    qb, kb, vb = inputs.qkv_bits(heads, kv, n, d, (5, 6, 7))
    grow = np.repeat(1.0 + 0.8 * np.arange(-(-n // B)), B)[:n].astype(np.float32)
    kf = inputs.bf16_bits_to_f32(kb) * grow[None, :, None]
    qf = np.abs(inputs.bf16_bits_to_f32(qb))
    kf = np.abs(kf)                      # positive scores that grow with the key block
    kb = inputs.f32_to_bf16_bits(kf)
    qb = inputs.f32_to_bf16_bits(qf * 0.5)
    # halve V so |o| stays below 4, where bf16 output still resolves 1e-2
    vb = inputs.f32_to_bf16_bits(inputs.bf16_bits_to_f32(vb) * 0.5)
    from gpu_common import to_device_bf16
    q, k, v = to_device_bf16(qb), to_device_bf16(kb), to_device_bf16(vb)
    o, lse = bsa.attention(q, k, v, lay, scale)
    torch.cuda.synchronize()
    bsa.bsa_get_status(lay.handle)
    sets = OL.kept_sets(kind, n, B, L, **pat)
    o_ref, lse_ref = _oracle((qb, kb, vb), sets, B, scale)
    # row maxima span many multiples of the kernel's rescale threshold (8 in
    # exp2 units, about 5.5 in lse units): the rescale path is really taken
    assert float(np.nanmax(lse_ref) - np.nanmin(lse_ref[np.isfinite(lse_ref)])) > 40
    assert_close(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "rescale")
    lay.close()


def test_large_scale_rescales():
    """A large softmax scale makes row maxima jump far beyond the rescale
    threshold between blocks; V is halved so |o| stays where bf16 resolves 1e-2."""
    n, B, d = 2048, 64, 128
    pat = dict(window=2, global_first=1, dyadic_kmin=2)
    lay = bsa.Layout(OL.DYADIC, n, B, 1, torch.cuda.current_device(), **pat)
    qb, kb, vb = inputs.qkv_bits(4, 2, n, d)
    vb = inputs.f32_to_bf16_bits(inputs.bf16_bits_to_f32(vb) * 0.5)
    from gpu_common import to_device_bf16
    o, lse = bsa.attention(to_device_bf16(qb), to_device_bf16(kb), to_device_bf16(vb), lay, 1.5)
    torch.cuda.synchronize()
    bsa.bsa_get_status(lay.handle)
    sets = OL.kept_sets(OL.DYADIC, n, B, 1, **pat)
    o_ref, lse_ref = _oracle((qb, kb, vb), sets, B, 1.5)
    assert_close(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "scale 1.5")
    lay.close()


# ----------------------------------------------------------------- full size
FULL = ["band_global_32k", "bf1_dyadic_gqa_32k", "static_random_131k"]


def _head_errors(w, qb, kb, vb, sets, o, lse, f, rows=None):
    """(max|do|, sum|do|, count, max|dlse|, sum|dlse|) of head f against the
    oracle, over every query block (or the blocks in ``rows``)."""
    g = w.heads // w.kv_heads
    scale = default_scale(w.d)
    qf = inputs.bf16_bits_to_f64(qb[f:f + 1])
    kf = inputs.bf16_bits_to_f64(kb[f // g:f // g + 1])
    vf = inputs.bf16_bits_to_f64(vb[f // g:f // g + 1])
    lay1 = [sets[f % w.layout_heads]]
    o_g = o[f].float().cpu().numpy().astype(np.float64)
    l_g = lse[f].cpu().numpy().astype(np.float64)
    mo = so = ml = sl = 0.0
    cnt = lcnt = 0
    for i in (range(w.n_blocks) if rows is None else rows):
        t0, t1 = i * w.B, min(w.n, (i + 1) * w.B)
        o_ref, lse_ref = OA.forward_block_rows(qf, kf, vf, lay1, w.B, scale, 0, i)
        do = np.abs(o_g[t0:t1] - o_ref)
        dl = np.abs(l_g[t0:t1] - lse_ref)
        mo, so, cnt = max(mo, float(do.max())), so + float(do.sum()), cnt + do.size
        ml, sl, lcnt = max(ml, float(dl.max())), sl + float(dl.sum()), lcnt + dl.size
    return mo, so, cnt, ml, sl, lcnt


@pytest.mark.parametrize("name", FULL)
def test_full_size_elementwise(name):
    """The benchmark's launch on the full workload against the oracle, element
    by element: every head and query block of the two 32K workloads; on the
    131K random workload two whole heads (the first and the last) and the
    longest row of every other head."""
    w = WORKLOADS[name]
    lay = bsa.Layout.for_workload(w, torch.cuda.current_device())
    (qb, kb, vb), (q, k, v) = device_inputs(w.heads, w.kv_heads, w.n, w.d)
    o, lse = bsa.attention(q, k, v, lay, default_scale(w.d))
    torch.cuda.synchronize()
    bsa.bsa_get_status(lay.handle)
    sets = OL.kept_sets_for(w)
    if name == "static_random_131k":
        plan = {0: None, w.heads - 1: None}
        for f in range(1, w.heads - 1):
            lens = [len(r) for r in sets[f % w.layout_heads]]
            plan[f] = [int(np.argmax(lens))]
    else:
        plan = {f: None for f in range(w.heads)}
    mo = so = ml = sl = 0.0
    cnt = lcnt = 0
    for f, rows in plan.items():
        a, b, c, d_, e, f_ = _head_errors(w, qb, kb, vb, sets, o, lse, f, rows)
        mo, so, cnt, ml, sl, lcnt = max(mo, a), so + b, cnt + c, max(ml, d_), sl + e, lcnt + f_
    assert mo <= MAX_ABS_TOL and so / cnt <= MEAN_ABS_TOL, (name, "o", mo, so / cnt)
    assert ml <= MAX_ABS_TOL and sl / lcnt <= MEAN_ABS_TOL, (name, "lse", ml, sl / lcnt)
    assert torch.isfinite(lse).all() and torch.isfinite(o.float()).all()
    lay.close()


# ----------------------------------------------------------------- invariants
def test_dropped_blocks_and_future_tokens_bitwise():
    n, B, d = 2048, 128, 128
    pat = dict(window=1, global_first=1)
    lay = bsa.Layout(OL.BAND_GLOBAL, n, B, 1, torch.cuda.current_device(), **pat)
    _, (q, k, v) = device_inputs(2, 2, n, d)
    o1, l1 = bsa.attention(q, k, v, lay)
    # block 5 is kept only by query blocks 5 and 6 (band width 1, plus block 0)
    k2, v2 = k.clone(), v.clone()
    k2[:, 5 * B:6 * B] += 3.0
    v2[:, 5 * B:6 * B] -= 2.0
    o2, l2 = bsa.attention(q, k2, v2, lay)
    torch.cuda.synchronize()
    untouched = [i for i in range(n // B) if i not in (5, 6)]
    for i in untouched:
        sl = slice(i * B, (i + 1) * B)
        assert torch.equal(o1[:, sl], o2[:, sl]) and torch.equal(l1[:, sl], l2[:, sl])
    assert not torch.equal(o1[:, 5 * B:7 * B], o2[:, 5 * B:7 * B])
    # future tokens: rows t <= 700 cannot see K/V at u > 700
    k3, v3 = k.clone(), v.clone()
    k3[:, 701:] = 7.0
    v3[:, 701:] = -7.0
    o3, l3 = bsa.attention(q, k3, v3, lay)
    torch.cuda.synchronize()
    assert torch.equal(o1[:, :701], o3[:, :701]) and torch.equal(l1[:, :701], l3[:, :701])
    lay.close()


def test_run_to_run_bitwise_deterministic():
    w = WORKLOADS["bf1_dyadic_gqa_32k"]
    n = 8192
    lay = bsa.Layout(w.pattern.kind, n, w.B, 1, torch.cuda.current_device(),
                     window=2, global_first=1, dyadic_kmin=2)
    _, (q, k, v) = device_inputs(8, 4, n, 128)
    o1, l1 = bsa.attention(q, k, v, lay)
    o2, l2 = bsa.attention(q, k, v, lay)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    lay.close()


def test_concurrent_forwards_on_one_layout():
    # Forwards sharing a layout on different streams, overlapping on the GPU,
    # each claim their own work counter: every result equals the serial one.
    n, B, d = 8192, 64, 128
    dev = torch.cuda.current_device()
    lay = bsa.Layout(OL.DYADIC, n, B, 1, dev, window=2, global_first=1, dyadic_kmin=2)
    _, (q, k, v) = device_inputs(8, 4, n, d)
    o_ref, l_ref = bsa.attention(q, k, v, lay)
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in range(4)]
    outs = []
    for rep in range(3):
        for s in streams:
            with torch.cuda.stream(s):
                outs.append(bsa.attention(q, k, v, lay, stream=s))
    torch.cuda.synchronize()
    for o, l in outs:
        assert torch.equal(o, o_ref) and torch.equal(l, l_ref)
    bsa.bsa_get_status(lay.handle)
    lay.close()


def test_more_calls_in_flight_than_work_counters():
    """136 forwards and 8 backwards on one layout, spread over 8 streams in a
    seeded random order and enqueued without waiting, more calls than the
    layout has work counters (64): calls that come back to a counter are
    ordered behind its previous user, so every output equals the serial one
    bit for bit (dq too: it is accumulated without atomics)."""
    n, B, d, heads, kv = 4096, 64, 128, 8, 4
    dev = torch.cuda.current_device()
    lay = bsa.Layout(OL.DYADIC, n, B, 1, dev, window=2, global_first=1, dyadic_kmin=2)
    _, (q, k, v) = device_inputs(heads, kv, n, d)
    dout = torch.randn(heads, n, d, device="cuda", generator=torch.Generator("cuda").manual_seed(5)).to(torch.bfloat16)
    o_ref, l_ref = bsa.attention(q, k, v, lay)
    dq_ref, _, _ = bsa.attention_backward(q, k, v, o_ref, l_ref, dout, lay)
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in range(8)]
    rng = np.random.default_rng(64)
    fwd, bwd = [], []
    for c in range(144):
        s = streams[int(rng.integers(8))]
        with torch.cuda.stream(s):
            if c % 18 == 17:
                bwd.append(bsa.attention_backward(q, k, v, o_ref, l_ref, dout, lay, stream=s)[0])
            else:
                fwd.append(bsa.attention(q, k, v, lay, stream=s))
    torch.cuda.synchronize()
    assert len(fwd) == 136 and len(bwd) == 8
    for o, l in fwd:
        assert torch.equal(o, o_ref) and torch.equal(l, l_ref)
    for dq in bwd:
        assert torch.equal(dq, dq_ref)
    bsa.bsa_get_status(lay.handle)
    lay.close()


# ----------------------------------------------------------------- boundary
def test_invalid_arguments_launch_nothing():
    n, B, d = 1024, 64, 128
    dev = torch.cuda.current_device()
    lay = bsa.Layout(OL.DYADIC, n, B, 1, dev, window=2, global_first=1)
    _, (q, k, v) = device_inputs(2, 1, n, d)
    o = torch.full_like(q, 5.0)
    lse = torch.full((2, n), 5.0, device="cuda")
    h = lay.handle

    def bad(status, **over):
        a = dict(q=q, k=k, v=v, layout=h, B=B, n=n, heads=2, kv_heads=1, d=d, scale=0.1, o=o, lse=lse)
        a.update(over)
        with pytest.raises(bsa.BsaError) as ei:
            bsa.bsa_forward(**a)
        assert ei.value.status == status, (over, ei.value)

    bad(2, B=128)
    bad(2, n=n - 1)
    bad(3, d=96)
    bad(2, heads=3, kv_heads=2)
    bad(1, scale=0.0)
    bad(1, scale=float("nan"))
    bad(1, q=q.data_ptr() + 2)
    bad(1, o=0)
    bad(1, lse=lse.data_ptr() + 1)
    torch.cuda.synchronize()
    assert torch.all(o.float() == 5.0) and torch.all(lse == 5.0)
    bsa.bsa_get_status(h)
    lay.close()


def test_bounded_wait_reports_timeout_and_context_survives():
    n, B, d = 1024, 128, 128
    dev = torch.cuda.current_device()
    lay = bsa.Layout(OL.BAND_GLOBAL, n, B, 1, dev, window=1, global_first=1)
    bsa.bsa_debug_timeout_probe(lay.handle, d, 2_000_000)        # 2 ms limit
    with pytest.raises(bsa.BsaError) as ei:
        bsa.bsa_get_status(lay.handle)
    assert ei.value.status == 7
    bsa.bsa_get_status(lay.handle)                                 # cleared
    # the context is still healthy: a normal forward is correct afterwards
    (qb, kb, vb), (q, k, v) = device_inputs(1, 1, n, d)
    o, lse = bsa.attention(q, k, v, lay)
    torch.cuda.synchronize()
    bsa.bsa_get_status(lay.handle)
    o_ref, lse_ref = _oracle((qb, kb, vb), OL.kept_sets(OL.BAND_GLOBAL, n, B, 1, window=1, global_first=1),
                             B, default_scale(d))
    assert_close(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "after timeout")
    lay.close()
