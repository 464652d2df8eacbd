"""The rounding allowance the GPU parity tests give a bf16 output: half the
gap between bf16 neighbours at the rounded value.  Checked on the CPU against
torch's own fp32 -> bf16 rounding (round to nearest even), including values
on both sides of powers of two and exact midpoints, where the bound is met
with equality."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from gpu_common import bf16_half_ulp


def _round_bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def test_half_ulp_bounds_round_to_nearest():
    rng = np.random.default_rng(7)
    c = np.concatenate([
        rng.standard_normal(200_000) * 10.0 ** rng.uniform(-6, 4, 200_000),
        # just below and just above powers of two, both signs
        np.ldexp(1.0, np.arange(-20, 20)) * (1 - 2.0 ** -10),
        np.ldexp(1.0, np.arange(-20, 20)) * (1 + 2.0 ** -10),
        -np.ldexp(1.0, np.arange(-20, 20)) * (1 - 2.0 ** -12),
    ]).astype(np.float32).astype(np.float64)
    got = _round_bf16(c)
    err = np.abs(got - c)
    assert np.all(err <= bf16_half_ulp(got))
    # tight: the worst sample sits close to half a gap
    assert (err / bf16_half_ulp(got)).max() > 0.99


def test_half_ulp_at_midpoints_and_known_values():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties go to even (1.0), a
    # move of exactly half the gap 2^-7
    c = np.array([1 + 2.0 ** -8, 256 + 1.0, 3 * 2.0 ** -8 + 1])
    got = _round_bf16(c)
    assert np.array_equal(got, [1.0, 256.0, 1 + 2.0 ** -6])
    assert np.array_equal(np.abs(got - c), bf16_half_ulp(got))
    assert np.array_equal(bf16_half_ulp([1.0, 1.5, 255.0, 256.0, -300.0]),
                          [2.0 ** -8, 2.0 ** -8, 0.5, 1.0, 1.0])
