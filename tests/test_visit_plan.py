"""The prefill kernels' tile schedule, run on the host (the same make_plan /
visit_at code the kernels use, exported as a test hook): for query tiles of
sequences with and without a query offset, local windows, sliding windows and
group sizes, every visible (row, key) pair is claimed by exactly one visit on
the branch the method routes it to, and nothing else is claimed."""
import ctypes

import numpy as np
import pytest

BN = BM = 128


def _visits(lib, L, Lk, w0, W, G, qt):
    cap = 4096
    buf = (ctypes.c_int * (5 * cap))()
    n = lib.jl_debug_prefill_visits(L, Lk, w0, W, G, qt, buf, cap)
    assert 0 <= n <= cap
    return np.array(buf[:5 * n], dtype=np.int64).reshape(n, 5)


def _check_tile(lib, L, Lk, w0, W, G, qt):
    off = Lk - L
    i0, i1 = qt * BM, min(qt * BM + BM - 1, L - 1)
    p = off + np.arange(i0, i1 + 1)[:, None]              # row positions
    visits = _visits(lib, L, Lk, w0, W, G, qt)
    nkt = max(int(visits[:, 0].max()) + 1 if len(visits) else 0, (Lk + BN - 1) // BN)
    j = np.arange(nkt * BN)[None, :]
    d = p - j
    visible = (d >= 0) & (j < Lk) & ((d < W) if W > 0 else True)
    grouped_expected = (G > 1) & (d >= w0)
    claims = np.zeros(d.shape, dtype=np.int64)
    grouped = np.zeros(d.shape, dtype=bool)
    for kt, grp, mask, lo, hi in visits:
        cols = slice(kt * BN, kt * BN + BN)
        dd = d[:, cols]
        keep = np.ones(dd.shape, dtype=bool) if not mask else (dd >= lo) & (dd <= hi)
        claims[:, cols] += keep
        grouped[:, cols] |= keep & bool(grp)
    assert np.array_equal(claims, visible.astype(np.int64)), (L, Lk, w0, W, G, qt)
    assert np.array_equal(grouped[visible], grouped_expected[visible]), (L, Lk, w0, W, G, qt)
    # the order the kernels rely on: every base visit before every grouped
    # one (the query tile is rotated in place between the two phases), and
    # the grouped visits on consecutive key tiles in ascending order (the key
    # correction advances its rotation by one tile per grouped visit)
    g = visits[:, 1]
    if len(g):
        assert np.all(np.diff(g) >= 0), (L, Lk, w0, W, G, qt)
        gk = visits[g == 1, 0]
        assert np.array_equal(gk, np.arange(gk[0], gk[0] + len(gk)) if len(gk) else gk), (L, Lk, w0, W, G, qt)


def _lib():
    from zero_shot_rope_b200 import build, jetlong
    build.build()
    lib = jetlong.lib()
    lib.jl_debug_prefill_visits.restype = ctypes.c_int
    lib.jl_debug_prefill_visits.argtypes = [ctypes.c_int] * 6 + [ctypes.POINTER(ctypes.c_int), ctypes.c_int]
    return lib


@pytest.mark.parametrize("G", [1, 2, 3, 5])
def test_schedule_claims_every_visible_pair_once(G):
    lib = _lib()
    rng = np.random.default_rng(G)
    for _ in range(60):
        L = int(rng.integers(1, 700))
        Lk = L + int(rng.choice([0, 0, 1, 127, 128, 129, int(rng.integers(1, 900))]))
        w0 = int(rng.choice([0, 1, 50, 127, 128, 129, 300, 10000]))
        W = int(rng.choice([0, 0, 1, 7, 64, 128, 129, 200, 513, 5000]))
        for qt in range((L + BM - 1) // BM):
            _check_tile(lib, L, Lk, w0, W, G, qt)


def test_schedule_rejects_bad_arguments():
    lib = _lib()
    buf = (ctypes.c_int * 5)()
    assert lib.jl_debug_prefill_visits(0, 10, 4, 0, 2, 0, buf, 1) == -1
    assert lib.jl_debug_prefill_visits(10, 5, 4, 0, 2, 0, buf, 1) == -1
    assert lib.jl_debug_prefill_visits(100, 100, 4, 0, 2, 1, buf, 1) == -1
    assert lib.jl_debug_prefill_visits(100, 100, -1, 0, 2, 0, buf, 1) == -1
