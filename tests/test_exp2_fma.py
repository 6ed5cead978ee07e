"""Accuracy of the FMA-pipe exp2 used by the forward softmax for part of its probabilities.

The device routine (exp2_fma2 in the kernels' PTX helper header) is Cody and Waite
range reduction plus a degree-4 polynomial for 2^f on [-1/2, 1/2].  This test reads
its constants from the source, replays every step in float32 arithmetic on the
host (each fused multiply-add rounded once), and checks the result against 2^x in
float64: relative error below 3e-6 wherever 2^x is a normal float, +0 below 2^-127
and for -inf.  CPU only.
"""
import os
import re

import numpy as np

HEADER = os.path.join(os.path.dirname(__file__), "..", "exact_io_aware_54_b200", "csrc", "ptx.cuh")


def _constants():
    src = open(HEADER).read()
    c = {}
    for name in ("kExp2C0", "kExp2C1", "kExp2C2", "kExp2C3", "kExp2C4", "kExp2Round"):
        m = re.search(r"constexpr float %s = ([0-9.eE+-]+)f;" % name, src)
        assert m, name
        c[name] = np.float32(float(m.group(1)))
    assert "<< 23) + 0x3f800000u" in src
    return c


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_fma_model(x):
    c = _constants()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-127.0))
    t = (x + c["kExp2Round"]).astype(np.float32)
    n = (t - c["kExp2Round"]).astype(np.float32)
    f = _fma32(n, np.full_like(n, -1.0), x)
    p = _fma32(np.full_like(f, c["kExp2C4"]), f, np.full_like(f, c["kExp2C3"]))
    for k in ("kExp2C2", "kExp2C1", "kExp2C0"):
        p = _fma32(p, f, np.full_like(f, c[k]))
    bits = ((t.view(np.uint32).astype(np.uint64) << 23) + 0x3F800000) & 0xFFFFFFFF
    two_n = bits.astype(np.uint32).view(np.float32)
    with np.errstate(under="ignore"):
        return (p.astype(np.float64) * two_n.astype(np.float64)).astype(np.float32)


def test_relative_error_on_normal_range():
    x = np.concatenate([np.linspace(-126.0, 12.0, 400001, dtype=np.float32),
                        np.float32(np.random.default_rng(54).uniform(-30, 10, 200000))])
    y = exp2_fma_model(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1)
    assert rel.max() < 3e-6, rel.max()


def test_integers_and_halves():
    # at integer x the polynomial sees f = 0, at x + 1/2 the interval edge
    x = np.arange(-126, 12, dtype=np.float32)
    for off in (0.0, 0.5, -0.5, 0.25):
        xs = (x + np.float32(off)).astype(np.float32)
        rel = np.abs(exp2_fma_model(xs).astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1)
        assert rel.max() < 3e-6, (off, rel.max())


def test_flush_to_zero_and_minus_infinity():
    x = np.array([-np.inf, -1e30, -1000.0, -200.0, -127.0, -126.6], dtype=np.float32)
    assert np.all(exp2_fma_model(x) == 0.0)
    # just above the flush point the value is tiny and never negative or NaN
    y = exp2_fma_model(np.array([-126.4, -126.0, -125.0], dtype=np.float32))
    assert np.all(np.isfinite(y)) and np.all(y > 0) and np.all(y < 2.0 ** -124)


def test_model_is_monotone_on_a_fine_grid():
    x = np.linspace(-20.0, 8.0, 200001, dtype=np.float32)
    y = exp2_fma_model(x)
    assert np.all(np.diff(y.astype(np.float64)) >= -1e-6 * y[1:].astype(np.float64))
