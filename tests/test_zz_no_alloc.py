"""The allocation-free forward entry point, bsa_forward_noalloc (GPU).

It serves callers that cannot allocate device memory -- a process whose GPU
memory was reserved up front by a serving framework's own pool, or a host
application that lends this library only the buffers it passes in, and code
that must not call cudaMalloc while running because it can synchronise the
device.  Such a caller builds its layout host-only (device = -1) and this
entry point stages the layout in the library's static device block.

Checked through the C ABI: two calls in a row on a host-only layout give the
same o and lse as bsa_forward on a device layout (within the parity
tolerance), the second call takes no device memory, the status word reads
clear after each call, a layout too large for the static block is refused
with a clear error, and so is a call on a stream that is capturing a graph.
This file is collected last so a failure here never hides the other tests'
results; it passes alone in a fresh process as well.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import block_sparse_long_bsa_b200 as bsa
from oracle import layouts as OL

from gpu_common import MAX_ABS_TOL, MEAN_ABS_TOL, device_inputs, default_scale

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    bsa.load_library()


def _close(a, b):
    d = (a.float() - b.float()).abs()
    return float(d.max()), float(d.mean())


@pytest.mark.parametrize("kind,n,B,L,heads,kv,d,pat", [
    (OL.DYADIC, 4096, 64, 1, 4, 2, 128, dict(window=2, global_first=1, dyadic_kmin=2)),
    (OL.RANDOM, 4096 - 40, 128, 2, 4, 4, 128, dict(density=0.2, seed=17)),
])
def test_noalloc_matches_bsa_forward_twice(kind, n, B, L, heads, kv, d, pat):
    dev = torch.cuda.current_device()
    dev_layout = bsa.Layout(kind, n, B, L, dev, **pat)
    host_layout = bsa.Layout(kind, n, B, L, -1, **pat)
    _, (q, k, v) = device_inputs(heads, kv, n, d)
    scale = default_scale(d)
    o_ref, lse_ref = bsa.attention(q, k, v, dev_layout, scale)
    torch.cuda.synchronize()
    bsa.bsa_get_status(dev_layout.handle)
    outs = [(torch.full_like(q, 3.0), torch.full((heads, n), 3.0, dtype=torch.float32, device="cuda"))
            for _ in range(2)]
    torch.cuda.synchronize()
    for call, (o, lse) in enumerate(outs):   # two calls in a row share the static block
        if call == 1:
            # the call's defining property: no device memory is taken, by the
            # library or through torch's caching allocator
            free0 = torch.cuda.mem_get_info()[0]
            allocs0 = torch.cuda.memory_stats().get("num_alloc_retries", 0), \
                torch.cuda.memory_stats().get("allocation.all.allocated", 0)
        bsa.bsa_forward_noalloc(q, k, v, host_layout.handle, B, n, heads, kv, d, scale, o, lse)
        torch.cuda.synchronize()
        if call == 1:
            assert torch.cuda.mem_get_info()[0] == free0
            assert (torch.cuda.memory_stats().get("num_alloc_retries", 0),
                    torch.cuda.memory_stats().get("allocation.all.allocated", 0)) == allocs0
        # the call's device status word (read through the host-only layout) is clear
        bsa.bsa_get_status(host_layout.handle)
        mo, ao = _close(o, o_ref)
        ml, al = _close(lse, lse_ref)
        assert mo <= MAX_ABS_TOL and ao <= MEAN_ABS_TOL, (mo, ao)
        assert ml <= MAX_ABS_TOL and al <= MEAN_ABS_TOL, (ml, al)
    dev_layout.close()
    host_layout.close()


def test_noalloc_refused_on_a_capturing_stream():
    """The layout is copied from host memory at every call, so a stream that is
    capturing a CUDA graph is refused before anything is enqueued."""
    n, B, d = 1024, 64, 128
    host_layout = bsa.Layout(OL.DYADIC, n, B, 1, -1, window=2, global_first=1, dyadic_kmin=2)
    _, (q, k, v) = device_inputs(2, 1, n, d)
    o = torch.empty_like(q)
    lse = torch.empty((2, n), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        g.capture_begin()
        try:
            with pytest.raises(bsa.BsaError) as ei:
                bsa.bsa_forward_noalloc(q, k, v, host_layout.handle, B, n, 2, 1, d, 0.125, o, lse, stream=s)
        finally:
            g.capture_end()
    assert ei.value.status == 3 and "capturing" in str(ei.value)
    torch.cuda.synchronize()
    host_layout.close()


def test_noalloc_refuses_layout_beyond_static_block():
    # 400,000 one-block rows: the work table and col_idx need 2,000,000 words,
    # more than the 1,048,576 the static block holds; refused before any copy
    n = 64 * 400_000
    big = bsa.Layout(OL.BAND_GLOBAL, n, 64, 1, -1, window=0, global_first=0)
    x = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(4, dtype=torch.float32, device="cuda")
    with pytest.raises(bsa.BsaError) as ei:
        bsa.bsa_forward_noalloc(x, x, x, big.handle, 64, n, 1, 1, 64, 0.125, x, lse)
    assert ei.value.status == 2 and "static scratch" in str(ei.value)
    big.close()
