"""FMA-pipe exp2 of the statistics kernel: the coefficient table matches its
generator, and the algorithm (range reduction, polynomial, exponent add)
keeps its stated error bound.  CPU only; the device function itself is held
against CUDA's exp2f in test_gpu_exp2.py."""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "cross_model_attention_block_b200", "csrc")
sys.path.insert(0, CSRC)
import gen_exp2_poly  # noqa: E402


def table():
    src = open(os.path.join(CSRC, "mf_sm100.cuh")).read()
    return np.array([float(v) for _, v in sorted(
        re.findall(r"constexpr float kExp2C(\d) = ([0-9.e+-]+)f;", src))], dtype=np.float32)


def exp2_emulated(x, c):
    """The device steps in float32 (Horner without fused rounding)."""
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic)).astype(np.float32)
    p = np.full_like(f, c[-1])
    for ck in c[-2::-1]:
        p = (p * f + ck).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def test_table_matches_generator():
    c, level = gen_exp2_poly.remez_exp2(4)
    np.testing.assert_array_equal(table(), c.astype(np.float32))
    assert level < 3e-6


def test_polynomial_levels_its_error():
    # a minimax fit equioscillates: degree + 2 alternating extrema of equal size
    c, level = gen_exp2_poly.remez_exp2(4)
    g = np.linspace(-0.5, 0.5, 200001)
    err = np.polyval(c[::-1], g) / np.exp2(g) - 1.0
    assert abs(np.max(np.abs(err)) - level) < 0.02 * level
    assert np.sum(np.diff(np.sign(err[np.abs(err) > 0.5 * level])) != 0) >= 5


def test_exp2_algorithm_error_bound():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-125, 0, 200000), -np.arange(126, dtype=np.float64),
                        -np.arange(125) - 0.5, [0.0, -1e-7, -0.49999, -0.50001]]).astype(np.float32)
    y = exp2_emulated(x, table()).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(y / ref - 1.0)) < 4e-6
    # below the clamp: a tiny normal number, never zero, never above 2^-124
    lo = exp2_emulated(np.array([-126.0, -200.0, -np.inf], np.float32), table())
    assert np.all(lo > 0) and np.all(lo < 2.0 ** -124)
