"""The append kernel's fp64 angle routine (rope_sincos in append_rope.cu),
checked on the CPU: its constants are read from the CUDA source and its steps
are replayed in exact rational arithmetic (each fma rounded once, as on the
GPU).  No GPU is needed; what the kernel computes from these steps is checked
end to end by the append parity tests."""
import math
import os
import re
from fractions import Fraction as F

import pytest

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "kv_cache_decode_rope_b200", "csrc", "append_rope.cu")


def _pi():
    """pi from Machin's formula, pi = 16 atan(1/5) - 4 atan(1/239), exactly
    summed to far below 2^-200."""
    def atan_inv(n):
        s, x2, t = F(0), F(1, n * n), F(1, n)
        for k in range(120):
            s += t / (2 * k + 1) * (1 if k % 2 == 0 else -1)
            t *= x2
        return s
    return 16 * atan_inv(5) - 4 * atan_inv(239)


def _constants():
    src = open(SRC).read()
    out = {}
    for name in ("kTwoOverPi", "kP1", "kP2", "kP3"):
        m = re.search(name + r"\s*=\s*(0x[0-9a-fA-Fp.+\-]+);", src)
        assert m, name
        out[name] = float.fromhex(m.group(1))
    return out


def _sig_bits(x: float) -> int:
    m, _ = math.frexp(abs(x))
    f = F(m)
    bits = 0
    while f.denominator != 1:
        f *= 2
        bits += 1
    return bits


def test_reduction_constants():
    c = _constants()
    half_pi = _pi() / 2
    # the two leading parts are short, so k * P1 and k * P2 are exact for |k| < 2^31
    assert _sig_bits(c["kP1"]) <= 22 and _sig_bits(c["kP2"]) <= 22
    total = F(c["kP1"]) + F(c["kP2"]) + F(c["kP3"])
    assert abs(total - half_pi) / half_pi < F(1, 10 ** 31)
    assert c["kTwoOverPi"] == float(2 / _pi())        # 2/pi rounded to nearest


def _fma(a, b, c):
    return float(F(a) * F(b) + F(c))


def _rope_sincos(x, c):
    """The kernel's steps, each fma rounded once."""
    k = float(round(x * c["kTwoOverPi"]))          # rint: ties to even, like Python's round
    r = _fma(-k, c["kP1"], x)
    r = _fma(-k, c["kP2"], r)
    r = _fma(-k, c["kP3"], r)
    r2 = r * r
    ps = -1.0 / math.factorial(19)
    for n in (17, 15, 13, 11, 9, 7, 5, 3):
        ps = _fma(ps, r2, (1.0 if (n // 2) % 2 == 0 else -1.0) / math.factorial(n))
    s_r = _fma(ps * r2, r, r)
    pc = 1.0 / math.factorial(20)
    for n in (18, 16, 14, 12, 10, 8, 6, 4, 2):
        pc = _fma(pc, r2, (1.0 if (n // 2) % 2 == 0 else -1.0) / math.factorial(n))
    c_r = _fma(pc, r2, 1.0)
    q = int(k) & 3
    sv, cv = (c_r, s_r) if q & 1 else (s_r, c_r)
    return (-sv if q & 2 else sv), (-cv if (q + 1) & 2 else cv)


def _ulp(x):
    return math.ulp(max(abs(x), 1e-300))


@pytest.mark.parametrize("scale", [1.0, 1e3, 131073.0, 2.0 ** 31 - 1])
def test_sincos_against_libm(scale):
    """Angles pos * base^(-2j/r) as the kernel forms them, up to positions
    near 2^31: within a few fp64 ulps of libm's sin and cos (absolute error
    scaled by 1, as the values are rotated vectors' coefficients)."""
    c = _constants()
    worst = 0.0
    for j in range(0, 64):
        inv = 2.0 ** (-2.0 * j / 128 * math.log2(10000.0))
        for frac in (0.0, 0.13, 0.5, 0.77, 1.0):
            pos = math.floor(scale * (0.5 + frac / 2))
            x = pos * inv
            s, co = _rope_sincos(x, c)
            worst = max(worst, abs(s - math.sin(x)), abs(co - math.cos(x)))
    assert worst <= 8 * 2.0 ** -53, worst


def test_sincos_quadrants_exact_points():
    c = _constants()
    for x, (es, ec) in [(0.0, (0.0, 1.0)), (math.pi / 2, (1.0, 0.0)), (math.pi, (0.0, -1.0)),
                        (3 * math.pi / 2, (-1.0, 0.0)), (-math.pi / 2, (-1.0, 0.0))]:
        s, co = _rope_sincos(x, c)
        assert abs(s - es) < 1e-15 and abs(co - ec) < 1e-15, (x, s, co)
