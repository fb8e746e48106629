"""The kernels' correction angle (cos, sin of n * inv_freq) against NumPy.

The kernels evaluate the sine and cosine of the correction rotation with their
own call-free fp64 routine (a two-step Cody–Waite reduction by pi/2 and Taylor
series) and round the result to fp32.  The test hook runs the same code on the
host; NumPy's fp64 cos / sin of the same fp64 product, rounded to fp32, must
agree to within one fp32 ulp everywhere and exactly almost everywhere.
"""
import ctypes

import numpy as np

import oracle


def _hook():
    from zero_shot_rope_b200 import build, jetlong

    build.build()
    f = jetlong.lib().jl_debug_angle_cs
    f.restype = None
    f.argtypes = [ctypes.c_int32, ctypes.c_double, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float)]
    return f


def _ulp_diff(a, b):
    a = np.asarray(a, dtype=np.float32).view(np.int32).astype(np.int64)
    b = np.asarray(b, dtype=np.float32).view(np.int32).astype(np.int64)
    return np.abs(a - b)


def test_angle_matches_numpy_fp64_rounded_to_fp32():
    f = _hook()
    rng = np.random.default_rng(7)
    ns = np.concatenate([np.arange(-300, 300), rng.integers(-(1 << 31) + 1, (1 << 31) - 1, 3000),
                         [131071, 98303, -98303, (1 << 31) - 1, -(1 << 31) + 1]]).astype(np.int64)
    c, s = ctypes.c_float(), ctypes.c_float()
    worst, exact, total = 0, 0, 0
    for theta, D in ((1e4, 64), (1e6, 128), (5e5, 128)):
        inv = oracle.rope_inv_freq(D, theta)
        for k in (0, 1, 5, D // 4, D // 2 - 1):
            for n in ns:
                f(int(n), float(inv[k]), ctypes.byref(c), ctypes.byref(s))
                ang = np.float64(n) * inv[k]
                want = (np.float32(np.cos(ang)), np.float32(np.sin(ang)))
                d = max(int(_ulp_diff(c.value, want[0])), int(_ulp_diff(s.value, want[1])))
                worst = max(worst, d)
                exact += d == 0
                total += 1
    assert worst <= 1, worst
    assert exact >= 0.999 * total, (exact, total)


def test_angle_special_values():
    f = _hook()
    c, s = ctypes.c_float(), ctypes.c_float()
    f(0, 1.0, ctypes.byref(c), ctypes.byref(s))
    assert c.value == 1.0 and s.value == 0.0      # R(0) is the identity, exactly
    for n in (1, 7, 1000, -3):
        f(n, 0.0, ctypes.byref(c), ctypes.byref(s))
        assert c.value == 1.0 and s.value == 0.0  # zero frequency
