"""The emulated 2^x of the tcgen05 prefill kernel, replayed step by step in
float32 on the CPU: its coefficients are the Remez fit, and over the whole
argument range the kernel can see its relative error stays far below bf16's
rounding (the probabilities are rounded to bf16 before the PV product)."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "paged_kv_cache_420_b200", "csrc")


def kernel_constants():
    text = open(os.path.join(CSRC, "prefill_tc.cuh")).read()
    c = [float(re.search(rf"kExp2C{i}\s*=\s*([0-9.eE+-]+)f", text).group(1)) for i in range(4)]
    magic = float(re.search(r"kRoundMagic\s*=\s*([0-9.eE+-]+)f", text).group(1))
    return np.array(c, dtype=np.float32), np.float32(magic)


def exp2_emulated(x):
    """The kernel's steps in float32: clamp, round by the magic add, cubic, exponent add."""
    c, magic = kernel_constants()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = np.float32(c[3]) * f + c[2]
    p = (p.astype(np.float32) * f + c[1]).astype(np.float32)
    p = (p * f + c[0]).astype(np.float32)
    bits = p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def test_coefficients_are_the_remez_fit():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    c_fit, err = mod.fit(3)
    c, _ = kernel_constants()
    np.testing.assert_array_equal(c, c_fit)
    assert err < 8e-5


def test_relative_error_over_the_argument_range():
    rng = np.random.default_rng(0)
    # the softmax argument is scaled score minus the lazily raised max: at most
    # the rescale slack (8) above zero, and anything below
    x = np.concatenate([np.linspace(-126, 8, 2_000_001, dtype=np.float32),
                        rng.uniform(-30, 8, 1_000_000).astype(np.float32),
                        np.arange(-126, 9, dtype=np.float32),           # integers: f = 0
                        np.arange(-126, 8, dtype=np.float32) + 0.5])    # ties of the rounding
    y = exp2_emulated(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    normal = x >= -125  # below, the result is subnormal (as good as 0, like ex2.approx.ftz)
    rel = np.abs(y[normal] / ref[normal] - 1)
    assert rel.max() < 8e-5, rel.max()
    assert 2.0 ** -9 > 10 * rel.max()  # an order of magnitude below bf16 rounding
    assert np.abs(y[~normal] - ref[~normal]).max() < 2.0 ** -135


def test_masked_scores_and_monotonicity():
    y = exp2_emulated(np.array([-np.inf, -1e30, -200.0, -126.0], dtype=np.float32))
    assert np.all(y >= 0) and np.all(y <= 2.0 ** -125)
    x = np.linspace(-20, 8, 100_001, dtype=np.float32)
    y = exp2_emulated(x)
    # monotone up to the fit's wiggle at the rounding boundaries
    assert np.all(np.diff(y.astype(np.float64)) / y[:-1] > -2e-4)
