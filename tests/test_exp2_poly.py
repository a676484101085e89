"""The FMA-pipe exp2 used for part of the attention softmax.

The kernel's constants must be the ones the committed generator produces
(Lawson's minimax fit of 2^f on [-1/2, 1/2]), and the full evaluation
(clamp, magic-number rounding, cubic, exponent add), replayed step by step in
float32, must stay within the error bound against exp2 over the range the
softmax uses (arguments <= 8 after the running-max shift).
"""
import os
import re
import runpy

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "learned_token_group_b200", "csrc")


def _kernel_coeffs():
    with open(os.path.join(CSRC, "ptx.cuh")) as f:
        text = f.read()
    m = re.search(r"kC0 = ([0-9.e+-]+)f, kC1 = ([0-9.e+-]+)f, kC2 = ([0-9.e+-]+)f, kC3 = ([0-9.e+-]+)f", text)
    assert m, "polynomial constants not found in ptx.cuh"
    return np.array([float(v) for v in m.groups()])


def _replay(t, c):
    """float32 replay of the device steps for one argument vector."""
    f32 = np.float32
    tc = np.maximum(t.astype(f32), f32(-126.0))
    r = (tc + f32(12582912.0)).astype(f32)
    n = (r - f32(12582912.0)).astype(f32)
    f = (tc - n).astype(f32)
    p = (f * f32(c[3]) + f32(c[2])).astype(f32)
    p = (p * f + f32(c[1])).astype(f32)
    p = (p * f + f32(c[0])).astype(f32)
    bits = p.view(np.int32) + (r.view(np.int32) << 23)
    return bits.astype(np.int32).view(f32)


def test_constants_match_generator():
    gen = runpy.run_path(os.path.join(CSRC, "exp2_poly.py"))
    c, err = gen["fit"]()
    assert err < 1e-4
    assert np.allclose(_kernel_coeffs(), c, rtol=1e-7, atol=0)


def test_error_bound_over_softmax_range():
    c = _kernel_coeffs()
    t = np.linspace(-125.0, 8.0, 2_000_001).astype(np.float32)
    got = _replay(t, c).astype(np.float64)
    ref = np.exp2(t.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1e-4, rel.max()


def test_underflow_and_masked_keys_are_tiny_not_nan():
    c = _kernel_coeffs()
    t = np.array([-np.inf, -1e30, -300.0, -127.0, -126.0], dtype=np.float32)
    got = _replay(t, c)
    assert np.isfinite(got).all() and (got >= 0).all() and (got < 2.0 ** -125).all()
