"""The entry points inside a CUDA graph: a forward, its gradients and a
selected-page decode step are captured once on torch's capture stream and
replayed after the inputs change in place.  Every call only enqueues work on
the stream it is given (no allocation, no synchronisation), so a replay must
give what an eager call on the same inputs gives: the forward, dq and the
decode bit for bit (their kernels are deterministic), dk and dv within the
fp32 reordering of their atomic sums.
"""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import block_sparse_long_bsa_b200 as bsa
from block_sparse_long_bsa_b200 import inputs
from oracle import decode as D
from oracle import layouts as OL

from gpu_common import to_device_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    bsa.load_library()


def test_forward_backward_decode_replay_in_a_cuda_graph():
    n, B, d, heads, kv = 2048, 64, 128, 4, 2
    scale = 1.0 / math.sqrt(d)
    pat = dict(window=2, global_first=1, dyadic_kmin=2)
    lay = bsa.Layout(OL.DYADIC, n, B, 1, torch.cuda.current_device(), **pat)
    qb, kb, vb = inputs.qkv_bits(heads, kv, n, d, seeds=(21, 22, 23))
    q, k, v = to_device_bf16(qb), to_device_bf16(kb), to_device_bf16(vb)
    do = to_device_bf16(inputs.normal_bf16_bits((heads, n, d), 24))
    # the decode step's cache: the same keys and values, paged in shuffled order
    order = np.random.default_rng(25).permutation(n // B)
    kcb, vcb, table = D.pages_from_sequences(kb, vb, 1, B, order)
    kc, vc = to_device_bf16(kcb), to_device_bf16(vcb)
    table = torch.from_numpy(table).cuda()
    pos = torch.tensor([n - 1], dtype=torch.int32, device="cuda")
    qd = q[:, n - 1].contiguous()

    # static outputs the graph writes
    o = torch.empty_like(q)
    lse = torch.empty((heads, n), dtype=torch.float32, device="cuda")
    dq = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    dk = torch.empty(k.shape, dtype=torch.float32, device="cuda")
    dv = torch.empty(v.shape, dtype=torch.float32, device="cuda")
    ws = torch.empty((heads, n), dtype=torch.float32, device="cuda")
    od = torch.empty_like(qd)
    lsed = torch.empty((heads,), dtype=torch.float32, device="cuda")

    def step():
        bsa.attention(q, k, v, lay, scale, o=o, lse=lse)
        bsa.attention_backward(q, k, v, o, lse, do, lay, scale, dq=dq, dk=dk, dv=dv, workspace=ws)
        bsa.decode(qd, kc, vc, table, pos, lay, 1, scale, o=od, lse=lsed)

    # eager calls first (one-time kernel attributes are set outside the capture)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    torch.cuda.synchronize()

    for seed in (31, 41):
        # new inputs in place, then the graph, then an eager reference run
        qb2, kb2, vb2 = inputs.qkv_bits(heads, kv, n, d, seeds=(seed, seed + 1, seed + 2))
        q.copy_(to_device_bf16(qb2))
        k.copy_(to_device_bf16(kb2))
        v.copy_(to_device_bf16(vb2))
        qd.copy_(q[:, n - 1])
        kcb2, vcb2, _ = D.pages_from_sequences(kb2, vb2, 1, B, order)
        kc.copy_(to_device_bf16(kcb2))
        vc.copy_(to_device_bf16(vcb2))
        graph.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in (o, lse, dq, dk, dv, od, lsed)]
        step()
        torch.cuda.synchronize()
        bsa.bsa_get_status(lay.handle)
        ref = (o, lse, dq, dk, dv, od, lsed)
        for name, a, b in zip(("o", "lse", "dq", "od", "lsed"), (got[0], got[1], got[2], got[5], got[6]),
                              (ref[0], ref[1], ref[2], ref[5], ref[6])):
            assert torch.equal(a, b), f"replay differs from eager on {name} (seed {seed})"
        for name, a, b in (("dk", got[3], ref[3]), ("dv", got[4], ref[4])):
            rel = float((a - b).norm() / b.norm())
            assert rel <= 1e-5, f"replay differs from eager on {name}: {rel:.2e} (seed {seed})"
    del graph
    lay.close()
