"""The attention's FMA-pipe exponential (ex2_poly2 in csrc/common.cuh) on the CPU: its four
coefficients are the float32 roundings of the degree-3 minimax polynomial for 2^f on
[-1/2, 1/2] that the Remez exchange in csrc/exp2_poly_coeffs.py derives, and the algorithm
(nearest-integer split by the 1.5 * 2^23 constant, Horner in float32, exponent added to the
bit pattern) holds a relative error below 1e-4 on [-125, 126] when carried out in float32.
The device evaluation is checked against the same bound by tests/test_gpu_parity.py."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "compressed_latent_space_b200", "csrc")


def _remez():
    spec = importlib.util.spec_from_file_location("exp2_poly_coeffs", os.path.join(CSRC, "exp2_poly_coeffs.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.remez_exp2()


def _source_coeffs():
    src = open(os.path.join(CSRC, "common.cuh")).read()
    body = src[src.index("void ex2_poly2("):]
    body = body[:body.index("\n}\n")]
    lines = [ln for ln in body.splitlines() if "fma2(" in ln and "p" in ln.split("=")[0]]
    nums = [float(v) for ln in lines for v in re.findall(r"(\d+\.\d+)f", ln)]
    # Horner order in the source: (c3, c2), c1, c0, each written twice (both halves)
    c3, c2, c1, c0 = nums[0], nums[2], nums[4], nums[6]
    return np.array([c0, c1, c2, c3], dtype=np.float32)


def _emulate(x, c):
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-125.0))
    j = (x + f32(12582912.0)).astype(f32)
    n = (j + f32(-12582912.0)).astype(f32)
    fr = (n * f32(-1.0) + x).astype(f32)
    p = (c[3] * fr + c[2]).astype(f32)
    p = (p * fr + c[1]).astype(f32)
    p = (p * fr + c[0]).astype(f32)
    bits = (p.view(np.uint32).astype(np.uint64) + (j.view(np.uint32).astype(np.uint64) << np.uint64(23))) & np.uint64(0xFFFFFFFF)
    return bits.astype(np.uint32).view(np.float32)


def test_source_coefficients_are_the_remez_solution():
    c, e = _remez()
    assert 7.0e-5 < e < 8.0e-5                      # degree 3 on a unit interval
    np.testing.assert_array_equal(_source_coeffs(), np.float32(c))


def test_remez_solution_equioscillates():
    c, e = _remez()
    f = np.linspace(-0.5, 0.5, 400001)
    err = (np.polyval(c[::-1], f) - np.exp2(f)) / np.exp2(f)
    assert abs(np.abs(err).max() - e) < 1e-9 * max(1.0, e) + 1e-12
    # five extrema of equal size and alternating sign (Chebyshev alternation for degree 3)
    segs = np.split(np.arange(len(f)), np.where(np.diff(np.sign(err)) != 0)[0] + 1)
    ext = np.array([err[s_[np.argmax(np.abs(err[s_]))]] for s_ in segs])
    assert len(ext) == 5
    assert np.all(np.abs(ext) > 0.999 * e) and np.all(ext[:-1] * ext[1:] < 0)


def test_float32_algorithm_error_bound():
    c = _source_coeffs()
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-125, 126, 2_000_000), np.arange(-125, 126.5, 0.5),
                        np.array([0.0, 0.4999999, -0.4999999, 1e-7, -1e-7])]).astype(np.float32)
    y = _emulate(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(y / ref - 1.0)) < 1e-4
    # below the clamp: about 2^-125 (the float16 probabilities it feeds round it to zero)
    y_low = _emulate(np.array([-126.0, -500.0, -np.inf], dtype=np.float32), c)
    assert np.all(y_low > 0) and np.all(y_low <= 2.0 ** -124.9)
