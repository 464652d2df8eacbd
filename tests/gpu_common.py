"""Shared helpers of the GPU parity tests: seeded inputs on the device, the
oracle on the same bf16 bits, and the parity tolerances (max and mean absolute error)."""
from __future__ import annotations

import math

import numpy as np

from block_sparse_long_bsa_b200 import inputs

# o and lse must match the fp64 oracle within these (max abs, mean abs) bounds.
MAX_ABS_TOL = 1e-2
MEAN_ABS_TOL = 1e-3


def to_device_bf16(bits: np.ndarray, device="cuda"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).to(device)


def device_inputs(heads, kv_heads, n, d, seeds=(0, 1, 2)):
    qb, kb, vb = inputs.qkv_bits(heads, kv_heads, n, d, seeds)
    return (qb, kb, vb), (to_device_bf16(qb), to_device_bf16(kb), to_device_bf16(vb))


def errors(o_gpu, lse_gpu, o_ref, lse_ref):
    """(max|do|, mean|do|, max|dlse|, mean|dlse|) over finite reference rows."""
    o = np.asarray(o_gpu, dtype=np.float64)
    lse = np.asarray(lse_gpu, dtype=np.float64)
    finite = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse), finite), "empty-row pattern differs"
    do = np.abs(o - o_ref)
    dl = np.abs(lse[finite] - lse_ref[finite]) if finite.any() else np.zeros(1)
    return float(do.max()), float(do.mean()), float(dl.max()), float(dl.mean())


def assert_close(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    mo, ao, ml, al = errors(o_gpu, lse_gpu, o_ref, lse_ref)
    big = float(np.abs(o_ref).max())
    assert mo <= MAX_ABS_TOL and ao <= MEAN_ABS_TOL, \
        f"{what}: o max {mo:.3e} mean {ao:.3e} (max |o_ref| {big:.2f})"
    assert ml <= MAX_ABS_TOL and al <= MEAN_ABS_TOL, f"{what}: lse max {ml:.3e} mean {al:.3e}"
    return mo, ao, ml, al


def default_scale(d):
    return 1.0 / math.sqrt(d)


def bf16_half_ulp(x):
    """Half the gap between neighbouring bf16 numbers at each value x (x itself
    a bf16 number): the most that rounding to nearest can have moved a real
    number whose rounded value is x.  bf16 keeps 8 significant bits, so for
    2^(e-1) <= |x| < 2^e the gap is 2^(e-8) and half of it 2^(e-9).  (A value
    just below 2^e that rounds up to 2^e moves by at most half the smaller gap
    below it, which is inside this bound too.)  Zero gets the bound of the
    smallest subnormal, 2^-134."""
    x = np.abs(np.asarray(x, dtype=np.float64))
    _, e = np.frexp(x)          # x = f 2^e with 1/2 <= f < 1
    return np.where(x > 0, np.ldexp(1.0, e - 9), 2.0 ** -134)
