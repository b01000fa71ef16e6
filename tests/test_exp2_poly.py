"""Error bound of the FMA-pipe exp2 used by the forward kernel's softmax.

The kernel evaluates 2^x as p(f) * 2^n with n = rint(x), f = x - n and a
cubic p fitted on [-1/2, 1/2]. Here the same float32 steps run in NumPy over
a dense grid and are compared with numpy.exp2: the relative error must stay
below 2e-4 (the bf16 rounding of the P operand it feeds is 2^-9 ~ 2e-3)."""
import numpy as np

C = [1.0, 0.6933686137199402, 0.24221783876419067, 0.05459282547235489]


def exp2_fma_numpy(x):
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    k = np.float32(12582912.0)
    t = (x + k).astype(np.float32)
    f = (x - (t - k)).astype(np.float32)
    p = np.float32(C[3])
    for c in (C[2], C[1], C[0]):
        p = (p * f + np.float32(c)).astype(np.float32)
    n = t.view(np.int32) - np.int32(0x4B400000)
    return (p.view(np.int32) + (n << 23)).view(np.float32)


def test_exp2_fma_relative_error():
    x = np.linspace(-120.0, 8.0, 2_000_001, dtype=np.float32)
    got = exp2_fma_numpy(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 2e-4, rel.max()


def test_exp2_fma_exact_at_integers():
    x = np.arange(-100, 9, dtype=np.float32)
    assert np.array_equal(exp2_fma_numpy(x), np.exp2(x.astype(np.float64)).astype(np.float32))


def test_generator_reproduces_coefficients():
    import importlib.util
    import os
    path = os.path.join(os.path.dirname(os.path.dirname(__file__)), "exact_tiled_attention_softmax_b200", "csrc",
                        "gen_exp2_poly.py")
    spec = importlib.util.spec_from_file_location("gen_exp2_poly", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    coeffs, err = mod.fit(3)
    assert np.allclose(np.float32(coeffs), np.float32(C), rtol=0, atol=0)
    assert err < 2e-4
