"""The polynomial exp2 of the prefill softmax (exp2_poly.cuh), pinned on the CPU.

The FP8 prefill kernels take one group of four exponentials in eight from a
cubic on the FMA pipes instead of the MUFU unit.  The coefficients are
written by csrc/exp2_poly.py (a Lawson minimax fit in relative error); these
tests check that the committed header is exactly what the script produces,
that the kernel's float32 steps (range reduction by the 1.5 * 2^23 rounding
constant, three fused multiply-adds, the exponent added as integer bits) stay
within 2e-4 relative error of exp2 over the whole input range the softmax
feeds it ([-126, 8]), and that the fit has the equal-ripple shape a minimax
fit must have.  The GPU side runs inside every FP8 parity test.
"""

import importlib.util
import os
import re

import numpy as np
import pytest

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "attention_flashattention_fwd_04_b200", "csrc")


def _script():
    spec = importlib.util.spec_from_file_location("exp2_poly_fit", os.path.join(CSRC, "exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _header_coefficients():
    with open(os.path.join(CSRC, "exp2_poly.cuh")) as f:
        text = f.read()
    found = dict(re.findall(r"kExp2C(\d)\s*=\s*([-+0-9.eE]+)f;", text))
    assert sorted(found) == ["0", "1", "2", "3"]
    return np.array([float(found[str(k)]) for k in range(4)], dtype=np.float32)


def _kernel_exp2(x, c32):
    """exp2_poly's steps in float32: clamp, round by the 1.5 * 2^23 constant,
    Horner with fused multiply-adds (one rounding each: the float32 product is
    exact in float64), then n added to the exponent field."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0)).astype(np.float32)).astype(np.float32)
    q = np.full_like(f, c32[3])
    for k in (2, 1, 0):
        q = (q.astype(np.float64) * f.astype(np.float64) + np.float64(c32[k])).astype(np.float32)
    bits = (q.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_header_is_the_scripts_fit_bit_for_bit():
    c32 = _script().fit().astype(np.float32)
    assert np.array_equal(c32.view(np.uint32), _header_coefficients().view(np.uint32))


def test_float32_steps_within_2e4_relative_on_the_softmax_range():
    c32 = _header_coefficients()
    x = np.linspace(-126.0, 8.0, 2_000_001)
    got = _kernel_exp2(x, c32).astype(np.float64)
    ref = np.exp2(x.astype(np.float32).astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() <= 2e-4
    # the script's own report agrees (it models the same steps)
    assert _script().report(c32) <= 2e-4


def test_exponent_shift_drops_the_rounding_constant():
    # bits(1.5 * 2^23) = 0x4B400000 has its low 9 bits clear, so shifting
    # bits(t) left by 23 is the same as shifting bits(t) - bits(1.5 * 2^23).
    assert (0x4B400000 << 23) & 0xFFFFFFFF == 0
    c32 = _header_coefficients()
    # f = 0: the result is 2^n * c0 exactly while it stays a normal number
    # (at n = -126 the exponent field reaches 0 and the bits read as a
    # subnormal; the range test above covers that point against the bound).
    for n in range(-125, 9):
        got = float(_kernel_exp2(np.array([float(n)]), c32)[0])
        assert got == float(c32[0]) * 2.0 ** n


def test_fit_equioscillates():
    # A degree-3 minimax fit in relative error touches its largest error at
    # five points with alternating signs and (nearly) equal size.
    c = _script().fit()
    f = np.linspace(-0.5, 0.5, 200_001)
    err = np.polyval(c[::-1], f) / np.exp2(f) - 1.0
    inner = np.where((np.diff(np.sign(np.diff(err))) != 0))[0] + 1
    ext = np.concatenate(([0], inner, [f.size - 1]))
    vals = err[ext]
    assert vals.size >= 5
    assert np.all(np.sign(vals[1:]) != np.sign(vals[:-1]))
    mags = np.abs(vals)
    assert mags.max() / mags.min() < 1.02
    assert mags.max() < 1.5e-4


@pytest.mark.parametrize("k, delta", [(0, 1e-3), (1, 2e-3), (2, 5e-3), (3, 1e-2)])
def test_a_perturbed_coefficient_breaks_the_bound(k, delta):
    c32 = _header_coefficients().copy()
    c32[k] = np.float32(c32[k] + delta)
    x = np.linspace(-20.0, 8.0, 200_001)
    rel = np.abs(_kernel_exp2(x, c32).astype(np.float64) - np.exp2(x)) / np.exp2(x)
    assert rel.max() > 2e-4
