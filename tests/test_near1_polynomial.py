"""The float32 kernels' retention near 1 (device_math.cuh, kNear1*): where
|delta A| < 2^-8 they take e^z = 1 + zl (c1 + zl c2), zl = z log2(e), rounded
once, instead of the SFU's exp2. CPU checks of its constants and of its error
over the band, with float32 arithmetic emulated exactly (each fused
multiply-add rounded once to float32). No GPU."""
import math
import os
import re

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
HEADER = os.path.join(os.path.dirname(HERE), "selective_state_space_51_b200",
                      "csrc", "device_math.cuh")


def _constants():
    text = open(HEADER).read()
    out = {}
    for name in ("kNear1Zl", "kNear1C1", "kNear1C2"):
        m = re.search(r"constexpr float %s = ([0-9.eE+-]+)f;" % name, text)
        assert m, name
        out[name] = np.float32(float(m.group(1)))
    return out


def _fma32(a, b, c):
    """float32 fused multiply-add: the product and sum exact in float64 for
    float32 operands of this size, then one rounding to float32."""
    return (a.astype(np.float64) * b.astype(np.float64)
            + c.astype(np.float64)).astype(np.float32)


def test_constants_are_the_series_coefficients():
    k = _constants()
    ln2 = math.log(2.0)
    assert k["kNear1C1"] == np.float32(ln2)
    assert k["kNear1C2"] == np.float32(ln2 * ln2 / 2)
    # the band: |z| < 2^-8, in units of zl = z / ln 2
    assert k["kNear1Zl"] == np.float32(2.0 ** -8 / ln2)


def test_polynomial_error_over_the_band():
    k = _constants()
    zl = np.linspace(-float(k["kNear1Zl"]), float(k["kNear1Zl"]), 400001,
                     dtype=np.float64).astype(np.float32)
    t = _fma32(zl, np.full_like(zl, k["kNear1C2"]),
               np.full_like(zl, k["kNear1C1"]))
    p = _fma32(zl, t, np.ones_like(zl))
    ref = np.exp2(zl.astype(np.float64))
    ulp = np.spacing(ref.astype(np.float32)).astype(np.float64)
    err = (p.astype(np.float64) - ref) / ulp
    # within 0.7 units in the last place (truncation |z|^3/6 < 0.17 ulp plus
    # the final rounding), with no bias that a held input could compound
    assert np.max(np.abs(err)) < 0.7
    assert abs(float(np.mean(err))) < 0.02


def test_held_input_retentions_are_correctly_rounded():
    """The retentions of a held tiny step (softplus(-12) ~ 6e-6, A = -1 ...
    -16): each polynomial value is the correctly rounded float32 of e^z, so
    a retention repeated over thousands of steps compounds no more error
    than any float32 exp would."""
    k = _constants()
    d = np.float32(np.log1p(np.exp(-12.0)))
    for n in range(1, 17):
        zl = np.float32(d * np.float32(-n * math.log2(math.e)))
        assert abs(zl) < k["kNear1Zl"]
        t = _fma32(np.array([zl]), np.array([k["kNear1C2"]]),
                   np.array([k["kNear1C1"]]))
        a = _fma32(np.array([zl]), t, np.array([np.float32(1.0)]))[0]
        exact = math.exp(float(zl) * math.log(2.0))
        assert a == np.float32(exact), n
