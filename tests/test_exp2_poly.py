"""The FMA-pipe 2^x of the attention kernels (exp2_poly2 in tcgen05.cuh).

The header's constants must be the ones exp2_poly_fit.py derives, and a
float32 emulation of the device steps (clamp, rounding by 1.5 * 2^23, Horner,
exponent-field add) must stay within the fit's relative error of 2^x over the
range the softmax loops use.
"""
import importlib.util
import os
import re

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "scratch_llama_decoder_b200", "csrc")


def _fit():
    spec = importlib.util.spec_from_file_location("exp2_poly_fit",
                                                  os.path.join(CSRC, "exp2_poly_fit.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _header_coefficients():
    src = open(os.path.join(CSRC, "tcgen05.cuh")).read()
    vals = {int(k): float(v) for k, v in re.findall(r"EXP2_C(\d) = ([0-9.eE+-]+)f", src)}
    return [vals[k] for k in sorted(vals)]


def _f32(x):
    return np.asarray(x, dtype=np.float32)


def _fma32(a, b, c):
    # a*b is exact in float64 for float32 operands; one rounding to float32 after the add
    return _f32(a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64))


def _exp2_poly_emulated(x, c):
    x = np.maximum(_f32(x), np.float32(-126.0))
    t = _f32(x + np.float32(12582912.0))
    k = _f32(t - np.float32(12582912.0))
    f = _fma32(k, _f32(-1.0), x)
    p = _fma32(_f32(c[3]), f, _f32(c[2]))
    p = _fma32(p, f, _f32(c[1]))
    p = _fma32(p, f, _f32(c[0]))
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_header_constants_match_fit():
    fit = _fit()
    assert _header_coefficients() == fit.coefficients()
    assert fit.horner_rel_error(fit.coefficients()) < 8e-5


def test_polynomial_is_minimax_on_the_interval():
    # equioscillation: the relative error reaches its bound (with alternating
    # sign) at deg + 2 points, and no other cubic through 2^0 = 1 does better
    fit = _fit()
    c = np.array(fit.remez(), dtype=np.float64)
    g = np.linspace(-0.5, 0.5, 20001)
    err = np.polyval(c[::-1], g) / np.exp2(g) - 1.0
    e = np.abs(err).max()
    assert 7e-5 < e < 8e-5
    # the Taylor cubic of 2^f at 0 is worse by more than a factor 5
    ln2 = np.log(2.0)
    taylor = np.array([1.0, ln2, ln2 ** 2 / 2, ln2 ** 3 / 6])
    et = np.abs(np.polyval(taylor[::-1], g) / np.exp2(g) - 1.0).max()
    assert et > 5 * e


def test_device_steps_error_bound():
    c = _header_coefficients()
    x = np.linspace(-125.0, 8.5, 2_000_001).astype(np.float32)
    y = _exp2_poly_emulated(x, c).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 8e-5
    # integer inputs: the polynomial at f = 0 times an exact power of two
    xi = np.arange(-125, 9).astype(np.float32)
    yi = _exp2_poly_emulated(xi, c).astype(np.float64)
    np.testing.assert_allclose(yi / np.exp2(xi.astype(np.float64)), np.float32(c[0]), rtol=1e-7)


def test_device_steps_below_range():
    c = _header_coefficients()
    x = np.array([-126.0, -127.5, -200.0, -1e6, -np.inf], dtype=np.float32)
    y = _exp2_poly_emulated(x, c)
    assert np.all(np.isfinite(y)) and np.all(y >= 0) and np.all(y < 2.0 ** -125)
