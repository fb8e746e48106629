"""The decode split plan on the host (the library's own planning code through
a test hook): for batches, head layouts, lengths and sliding windows, every
key a sequence attends to falls in exactly one split, and the workspace holds
every split's partial rows."""
import ctypes

import numpy as np
import pytest


def _lib():
    from zero_shot_rope_b200 import build, jetlong
    build.build()
    lib = jetlong.lib()
    lib.jl_debug_decode_plan.restype = ctypes.c_int
    lib.jl_debug_decode_plan.argtypes = [ctypes.c_int] * 7 + [ctypes.POINTER(ctypes.c_int),
                                                              ctypes.POINTER(ctypes.c_int),
                                                              ctypes.POINTER(ctypes.c_longlong)]
    return lib


def plan(lib, B, Hq, Hkv, D, M, W, bf16):
    ns, ch, rows = ctypes.c_int(), ctypes.c_int(), ctypes.c_longlong()
    assert lib.jl_debug_decode_plan(B, Hq, Hkv, D, M, W, bf16, ctypes.byref(ns), ctypes.byref(ch),
                                    ctypes.byref(rows)) == 0
    return ns.value, ch.value, rows.value


@pytest.mark.parametrize("bf16", [1, 0])
def test_every_attended_key_falls_in_one_split(bf16):
    lib = _lib()
    rng = np.random.default_rng(bf16)
    for _ in range(3000):
        B = int(rng.choice([1, 2, 3, 8, 17, 64, 300]))
        Hkv = int(rng.choice([1, 2, 4, 8]))
        Hq = Hkv * int(rng.choice([1, 2, 4, 8, 16]))
        D = int(rng.choice([64, 128]))
        M = int(rng.integers(1, 300000))
        W = int(rng.choice([0, 0, 1, 100, 4096, int(rng.integers(1, 300000))]))
        ns, ch, rows = plan(lib, B, Hq, Hkv, D, M, W, bf16)
        keys = min(M, W) if W > 0 else M
        assert ns >= 1 and ch >= 1
        assert ns * ch >= keys, (B, Hq, Hkv, D, M, W, ns, ch)     # no attended key left out
        assert (ns - 1) * ch < keys, (B, Hq, Hkv, D, M, W, ns, ch)  # no split past the keys
        assert ch % 64 == 0                                        # whole key tiles
        if bf16 and Hq // Hkv <= 8:  # the tensor-core decode: 256-key tiles at head_dim 64, 128 at 128
            assert ch % (256 if D == 64 else 128) == 0, (D, ch)
        assert rows >= B * Hq * ns, (B, Hq, Hkv, D, M, W, ns, rows)  # the workspace holds them


def test_plan_rejects_bad_sizes():
    lib = _lib()
    ns, ch, rows = ctypes.c_int(), ctypes.c_int(), ctypes.c_longlong()
    for args in ((0, 8, 2, 128, 10, 0, 1), (1, 6, 4, 128, 10, 0, 1), (1, 8, 2, 96, 10, 0, 1),
                 (1, 8, 2, 128, 0, 0, 1), (1, 8, 2, 128, 10, -1, 1)):
        assert lib.jl_debug_decode_plan(*args, ctypes.byref(ns), ctypes.byref(ch), ctypes.byref(rows)) == -1
