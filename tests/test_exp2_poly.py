"""The FMA-pipe exp2 used for part of the attention probabilities: its cubic and range
reduction, re-evaluated on the CPU in float32 from the constants in the CUDA header,
against numpy's exp2.  CPU only."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "block_sparse_attention_44_b200", "csrc", "fva_common.cuh")


def _consts():
    src = open(HDR).read()
    c = [float(re.search(rf"kExp2C{i}\s*=\s*([0-9.eE+-]+)f", src).group(1)) for i in range(4)]
    clamp = float(re.search(r"x = fmaxf\(x, (-?[0-9.]+)f\);", src).group(1))
    return np.float32(c), np.float32(clamp)


def exp2_poly_emulated(x):
    c, clamp = _consts()
    magic = np.float32(1.5 * 2 ** 23)
    x = np.maximum(np.asarray(x, dtype=np.float32), clamp)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic)).astype(np.float32)
    assert (np.abs(f) <= 0.5).all()
    p = (((c[3] * f + c[2]) * f + c[1]) * f + c[0]).astype(np.float32)
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-120.0, 8.0, 2_000_001, dtype=np.float32)
    got = exp2_poly_emulated(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 1.0e-4          # bf16 probabilities carry 2^-9 = 2e-3 relative steps


def test_underflow_region_stays_tiny_positive_and_finite():
    x = np.concatenate([np.linspace(-1e4, -100.0, 100_001, dtype=np.float32), np.float32([-np.inf])])
    y = exp2_poly_emulated(x)
    assert np.isfinite(y).all()
    assert (y >= 0).all() and (y < 1e-30).all()


def test_integer_points_and_monotone():
    k = np.arange(-100, 9, dtype=np.float32)
    assert np.allclose(exp2_poly_emulated(k), np.exp2(k), rtol=1e-4)
    x = np.linspace(-20.0, 8.0, 100_001, dtype=np.float32)
    y = exp2_poly_emulated(x)
    assert (np.diff(y.astype(np.float64)) >= -1e-6 * y[1:]).all()
