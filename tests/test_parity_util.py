"""The parity tests' output bound, pinned on the CPU: half an ulp of the
16-bit storage type is the largest error that rounding a value to that type
can make, and the bound reduces to 1e-2 where the storage rounding is below
it."""
import numpy as np

from exact_tiled_attention_softmax_b200 import workloads as W
from tests.parity_util import half_ulp, o_excess


def test_half_ulp_closed_forms():
    assert half_ulp(np.array([1.0]), "bf16")[0] == 2.0 ** -8
    assert half_ulp(np.array([3.0]), "bf16")[0] == 2.0 ** -7   # [2, 4): ulp 2^-6
    assert half_ulp(np.array([-5.0]), "bf16")[0] == 2.0 ** -6  # [4, 8): ulp 2^-5
    assert half_ulp(np.array([1.0]), "f16")[0] == 2.0 ** -11
    assert half_ulp(np.array([0.0]), "bf16")[0] == 2.0 ** -134
    assert half_ulp(np.array([1e-6]), "f16")[0] == 2.0 ** -25   # fp16 subnormal spacing 2^-24


def test_half_ulp_bounds_the_storage_rounding():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(200_000) * rng.choice([0.01, 1.0, 30.0], 200_000)).astype(np.float32)
    for storage, rounded in (("bf16", W.round_to_bf16(x)), ("f16", W.round_to_fp16(x))):
        err = np.abs(rounded.astype(np.float64) - x.astype(np.float64))
        assert np.all(err <= half_ulp(x, storage))
        # and it is tight: some value rounds by more than half of it
        assert np.any(err > 0.5 * half_ulp(x, storage))


def test_o_excess():
    want = np.array([0.5, 5.0, -3.0])
    got = want + np.array([0.009, 0.025, -0.017])
    # bf16 half ulps: 2^-9, 2^-6, 2^-7
    assert abs(o_excess(got, want) - (0.025 - 2.0 ** -6)) < 1e-12
    assert o_excess(np.zeros(0), np.zeros(0)) == 0.0
    # with the P-operand term: 2^-8 * p_abs more is allowed
    p_abs = np.array([0.0, 1.28, 0.0])
    assert abs(o_excess(got, want, p_abs=p_abs) - max(0.009 - 2.0 ** -9, 0.025 - 2.0 ** -6 - 0.005,
                                                      0.017 - 2.0 ** -7)) < 1e-12
