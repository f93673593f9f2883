"""The FMA-only erf and GELU' polynomials of the GEMM epilogues (csrc/gelu_poly.cuh),
checked on the CPU: the header is what its generator writes, and each polynomial,
evaluated in float32 with the header's own clamp, scale and coefficients, stays within
its stated error of scipy's erf and of Phi(x) + x phi(x) over the real line. The GPU
parity tests check the kernels' H against the oracle's exact-erf GELU to one bf16 ulp."""
import math
import os
import re

import numpy as np
from scipy.special import erf
from scipy.stats import norm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "vision_language_projector_b200", "csrc", "gelu_poly.cuh")
NUM = r"(-?[\d.]+(?:e-?\d+)?)"


def _functions():
    text = open(HEADER).read()
    out = {}
    for name, body in re.findall(r"uint64_t (\w+)\(float t0, float t1\) \{(.*?)\n\}", text, flags=re.S):
        lim = float(re.search(r"fmaxf\(t0, " + NUM + r"f\)", body).group(1))
        scale = float(re.search(r"f2_mul\(tc, tc\), f2_splat\(" + NUM + r"f\)", body).group(1))
        first = float(re.search(r"uint64_t p = f2_splat\(" + NUM + r"f\);", body).group(1))
        rest = [float(v) for v in re.findall(r"p = f2_fma\(p, s, f2_splat\(" + NUM + r"f\)\);", body)]
        out[name] = (abs(lim), scale, [first] + rest)
    return out


def _eval_f32(fn, t):
    lim, scale, coef = fn
    f = np.float32
    tc = np.clip(np.asarray(t, np.float32), f(-lim), f(lim))
    s = tc * tc * f(scale) - f(1.0)
    p = np.full_like(tc, f(coef[0]))
    for c in coef[1:]:
        p = p * s + f(c)
    return (tc * p).astype(np.float64)


def test_header_is_the_generators_output():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "gen", os.path.join(ROOT, "vision_language_projector_b200", "gen_gelu_poly.py"))
    gen = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    assert gen.render() == open(HEADER).read()


def test_both_polynomials_present():
    fns = _functions()
    assert set(fns) == {"erf_poly2", "dgelu_odd_poly2"}
    assert len(fns["erf_poly2"][2]) == 17 and len(fns["dgelu_odd_poly2"][2]) == 19


def test_erf_poly_error():
    fn = _functions()["erf_poly2"]
    t = np.linspace(-8.0, 8.0, 400001)
    err = np.abs(_eval_f32(fn, t) - erf(t))
    assert err.max() <= 2.5e-7
    np.testing.assert_array_equal(_eval_f32(fn, -t), -_eval_f32(fn, t))     # odd


def test_dgelu_poly_error():
    fn = _functions()["dgelu_odd_poly2"]
    x = np.linspace(-12.0, 12.0, 400001)
    got = 0.5 + _eval_f32(fn, x / math.sqrt(2.0))
    assert np.abs(got - (norm.cdf(x) + x * norm.pdf(x))).max() <= 3.5e-7


def test_gelu_from_the_poly_matches_the_exact_erf_gelu():
    fn = _functions()["erf_poly2"]
    x = np.linspace(-10.0, 10.0, 200001)
    g = 0.5 * x * (1.0 + _eval_f32(fn, x / math.sqrt(2.0)))
    assert np.abs(g - 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))).max() <= 2e-6
