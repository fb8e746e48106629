"""Pins for the fp64 CPU oracle (no GPU).

Each test ties the oracle to something other than itself: the worked G
examples, brute-force searches, closed forms, invariants the pages state,
textbook causal RoPE attention in the special cases where the method reduces
to it, and a pure-Python brute force on tiny inputs.  The planted-mistake tests
at the end check that plausible errors in the oracle are caught by these pins.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import bifocal as ob

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(12345)


# --------------------------------------------------------------------------
# Position policy
# --------------------------------------------------------------------------


def test_group_size_worked_examples():
    with open(os.path.join(GOLDEN, "group_size_examples.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        G = oracle.group_size(c["L"], c["w_pretrained"])
        assert G == c["G"], c
        if c["max_remote_position"] is not None:
            assert int(oracle.position_map(c["L"] - 1, G)) == c["max_remote_position"], c


def _smallest_sufficient_group(L, w):
    # brute force: the least g >= 1 such that g groups of w positions cover L
    g = 1
    while g * w < L:
        g += 1
    return g


@pytest.mark.parametrize("w", [1, 2, 7, 64, 256, 1000])
def test_group_size_is_least_sufficient_grouping(w):
    for L in range(0, 4000):
        assert oracle.group_size(L, w) == _smallest_sufficient_group(L, w)
    for L in RNG.integers(0, 1 << 20, size=200):
        assert oracle.group_size(int(L), w) == _smallest_sufficient_group(int(L), w)


def test_group_size_rejects_bad_arguments():
    with pytest.raises(ValueError):
        oracle.group_size(10, 0)
    with pytest.raises(ValueError):
        oracle.group_size(-1, 10)


@pytest.mark.parametrize("w", [3, 64, 256, 32768])
def test_remote_positions_stay_on_pretrained_grid(w):
    # The pages: every remote rotation angle stays on the model's pretrained
    # grid, with the least compression that achieves it.
    for L in list(range(1, 3 * w + 5, max(1, w // 16))) + [w * 4, w * 4 + 1, 131072]:
        G = oracle.group_size(L, w)
        assert int(oracle.position_map(L - 1, G)) <= w - 1
        if G > 1:  # one group less would leave the grid
            assert (L - 1) // (G - 1) > w - 1


def test_position_map_is_floor_division():
    for G in (1, 2, 3, 4, 5, 7):
        for x in range(0, 200):
            count = sum(1 for m in range(1, x + 1) if m % G == 0)  # multiples of G in [1, x]
            assert int(oracle.position_map(x, G)) == count


def test_correction_shift_values():
    p = np.arange(0, 50)
    for G in (1, 2, 3, 4):
        d = oracle.correction_shift(p, G)
        assert np.all(d <= 0)
        assert np.all(p + d == p // G)
    assert np.all(oracle.correction_shift(p, 1) == 0)


# --------------------------------------------------------------------------
# RoPE
# --------------------------------------------------------------------------


def test_inv_freq_closed_form():
    for D in (4, 64, 128):
        for theta in (1e4, 1e6):
            f = oracle.rope_inv_freq(D, theta)
            assert f.shape == (D // 2,)
            assert f[0] == 1.0
            # geometric with ratio theta^(-2/D): the pair after the last would be 1/theta
            ratio = f[1:] / f[:-1]
            assert np.allclose(ratio, theta ** (-2.0 / D), rtol=1e-13)
            assert math.isclose(f[-1] * theta ** (-2.0 / D), 1.0 / theta, rel_tol=1e-12)


def test_rope_matches_complex_exponential():
    # Independent formulation: pair k as the complex number x_k + i x_{k+D/2},
    # rotated by multiplication with exp(i m theta^(-2k/D)).
    D, theta = 16, 1e4
    x = RNG.standard_normal((50, D))
    m = RNG.integers(-3000, 3000, size=50)
    z = x[:, : D // 2] + 1j * x[:, D // 2:]
    k = np.arange(D // 2)
    zr = z * np.exp(1j * m[:, None] * theta ** (-2.0 * k / D))
    want = np.concatenate([zr.real, zr.imag], axis=1)
    assert np.allclose(oracle.rope_rotate(x, m, theta), want, atol=1e-12)


def test_rope_relative_position_property():
    D, theta = 32, 1e6
    q = RNG.standard_normal(D)
    k = RNG.standard_normal(D)
    for a, b in [(0, 0), (5, 3), (1000, 17), (70000, 131071), (3, 90000)]:
        lhs = oracle.rope_rotate(q, a, theta) @ oracle.rope_rotate(k, b, theta)
        rhs = oracle.rope_rotate(q, a - b, theta) @ k
        assert math.isclose(lhs, rhs, rel_tol=1e-9, abs_tol=1e-9)
        assert math.isclose(np.linalg.norm(oracle.rope_rotate(q, a, theta)), np.linalg.norm(q),
                            rel_tol=1e-13)


def test_correction_rotation_composes_additively():
    # Section 2 "Rotacao de Correcao On-the-Fly": R(delta(p)) R(p) = R(f(p)).
    D, theta = 128, 1e6
    x = RNG.standard_normal((256, D))
    p = np.concatenate([RNG.integers(0, 1 << 17, size=250), [0, 1, 4095, 4096, 131071, 98304]])
    for G in (1, 2, 3, 4, 5):
        lhs = oracle.rope_rotate(oracle.rope_rotate(x, p, theta), oracle.correction_shift(p, G), theta)
        rhs = oracle.rope_rotate(x, oracle.position_map(p, G), theta)
        assert np.max(np.abs(lhs - rhs)) < 1e-10


# --------------------------------------------------------------------------
# Attention: brute force, three routes, special cases
# --------------------------------------------------------------------------


def _raw_case(L, Hq, Hkv, D, seed):
    r = np.random.default_rng(seed)
    return (r.standard_normal((L, Hq, D)), r.standard_normal((L, Hkv, D)),
            r.standard_normal((L, Hkv, D)))


def _rotated(q_raw, k_raw, theta):
    L = q_raw.shape[0]
    pos = np.arange(L)
    qt = oracle.rope_rotate(q_raw, pos[:, None], theta)
    kt = oracle.rope_rotate(k_raw, pos[:, None], theta)
    return qt, kt


TINY = [  # (L, D, w_pretrained, w0): G = 1, 2, 3, 5 and window edge cases
    (1, 4, 1, 0), (2, 4, 1, 1), (5, 4, 2, 2), (9, 8, 3, 3), (17, 8, 4, 1),
    (23, 8, 5, 7), (30, 4, 6, 0), (40, 8, 8, 40), (33, 8, 11, 5), (26, 4, 26, 4),
]


@pytest.mark.parametrize("L,D,w_pre,w0", TINY)
def test_route_a_matches_pure_python_brute_force(L, D, w_pre, w0):
    theta = 1e4 if D == 8 else 500.0
    q_raw, k_raw, v = _raw_case(L, 1, 1, D, seed=L * 31 + w0)
    qt, kt = _rotated(q_raw, k_raw, theta)
    out, lse = oracle.bifocal_attention(qt, kt, v, [0, L], w_pre, w0, theta)
    bo, bl = oracle.brute_force_tiny(q_raw[:, 0].tolist(), k_raw[:, 0].tolist(), v[:, 0].tolist(),
                                     w_pre, w0, theta)
    assert np.max(np.abs(out[:, 0] - np.array(bo))) < 1e-11
    assert np.max(np.abs(lse[0] - np.array(bl))) < 1e-11


@pytest.mark.parametrize("L,w_pre,w0", [(64, 16, 8), (100, 30, 0), (97, 20, 13), (80, 80, 10),
                                        (128, 32, 128)])
def test_route_a_matches_raw_route_c(L, w_pre, w0):
    D, theta = 16, 1e4
    q_raw, k_raw, v = _raw_case(L, 4, 2, D, seed=L + w0)
    qt, kt = _rotated(q_raw, k_raw, theta)
    a_out, a_lse = oracle.bifocal_attention(qt, kt, v, [0, L], w_pre, w0, theta)
    c_out, c_lse = oracle.bifocal_attention_from_raw(q_raw, k_raw, v, L, w_pre, w0, theta)
    assert np.max(np.abs(a_out - c_out)) < 1e-10
    assert np.max(np.abs(a_lse - c_lse)) < 1e-10


@pytest.mark.parametrize("seqlens,w_pre,w0", [((70,), 20, 9), ((33, 64, 1), 16, 5),
                                              ((50, 50), 50, 0), ((90,), 25, 90)])
def test_route_a_matches_inclusion_exclusion_merge(seqlens, w_pre, w0):
    D, theta = 16, 1e4
    T = sum(seqlens)
    q, k, v = _raw_case(T, 4, 1, D, seed=T + w0)
    cu = np.concatenate([[0], np.cumsum(seqlens)])
    a_out, a_lse = oracle.bifocal_attention(q, k, v, cu, w_pre, w0, theta)
    b_out, b_lse = oracle.bifocal_attention_ie_merge(q, k, v, cu, w_pre, w0, theta)
    assert np.max(np.abs(a_out - b_out)) < 1e-10
    assert np.max(np.abs(a_lse - b_lse)) < 1e-10


@pytest.mark.parametrize("w0", [0, 1, 17, 1000])
def test_group_one_is_textbook_causal_rope(w0):
    # The pages: the method reproduces the base model exactly inside its native
    # context.  L <= w_pretrained gives G = 1, f = identity, delta = 0.
    L, D, theta = 120, 16, 1e6
    q, k, v = _raw_case(L, 4, 2, D, seed=7 + w0)
    out, lse = oracle.bifocal_attention(q, k, v, [0, L], 128, w0, theta)
    ref_o, ref_l = oracle.causal_rope_attention(q, k, v)
    assert np.max(np.abs(out - ref_o)) < 1e-13
    assert np.max(np.abs(lse - ref_l)) < 1e-13


@pytest.mark.parametrize("w_pre", [1, 3, 10])
def test_short_input_inside_window_is_textbook_causal_rope(w_pre):
    # L <= w0: every causal pair is local, whatever G is.
    L, D, theta = 60, 16, 1e4
    q, k, v = _raw_case(L, 2, 1, D, seed=w_pre)
    out, lse = oracle.bifocal_attention(q, k, v, [0, L], w_pre, L, theta)
    ref_o, ref_l = oracle.causal_rope_attention(q, k, v)
    assert np.max(np.abs(out - ref_o)) < 1e-13
    assert np.max(np.abs(lse - ref_l)) < 1e-13


@pytest.mark.parametrize("w_pre", [4, 9, 25])
def test_zero_window_is_causal_rope_at_grouped_positions(w_pre):
    # w0 = 0: every pair is remote, i.e. textbook RoPE attention with the
    # positions replaced by f(p).
    L, D, theta = 75, 16, 1e4
    q_raw, k_raw, v = _raw_case(L, 2, 2, D, seed=w_pre + 100)
    qt, kt = _rotated(q_raw, k_raw, theta)
    out, lse = oracle.bifocal_attention(qt, kt, v, [0, L], w_pre, 0, theta)
    G = oracle.group_size(L, w_pre)
    f = oracle.position_map(np.arange(L), G)[:, None]
    ref_o, ref_l = oracle.causal_rope_attention(oracle.rope_rotate(q_raw, f, theta),
                                                oracle.rope_rotate(k_raw, f, theta), v)
    assert np.max(np.abs(out - ref_o)) < 1e-10
    assert np.max(np.abs(lse - ref_l)) < 1e-10


def test_zero_queries_average_the_visible_values():
    # Closed form: with all scores equal, row i is the mean of V[0..i] and
    # lse = log(i + 1).
    L, D = 50, 8
    q = np.zeros((L, 2, D))
    _, k, v = _raw_case(L, 2, 1, D, seed=3)
    out, lse = oracle.bifocal_attention(q, k, v, [0, L], 10, 4, 1e4)
    mean = np.cumsum(v[:, 0], axis=0) / np.arange(1, L + 1)[:, None]
    assert np.max(np.abs(out[:, 0] - mean)) < 1e-13
    assert np.max(np.abs(lse[1] - np.log(np.arange(1, L + 1)))) < 1e-13


def test_rows_subset_and_varlen_independence():
    D, theta = 16, 1e4
    seqlens = (40, 1, 77)
    T = sum(seqlens)
    q, k, v = _raw_case(T, 2, 1, D, seed=99)
    cu = np.concatenate([[0], np.cumsum(seqlens)])
    full_o, full_l = oracle.bifocal_attention(q, k, v, cu, 16, 6, theta)
    rows = np.array([0, 5, 39, 40, 41, 60, 117])
    sub_o, sub_l = oracle.bifocal_attention(q, k, v, cu, 16, 6, theta, rows=rows)
    assert np.array_equal(sub_o, full_o[rows]) and np.array_equal(sub_l, full_l[:, rows])
    # each sequence is attended on its own
    o2, _ = oracle.bifocal_attention(q[41:], k[41:], v[41:], [0, 77], 16, 6, theta)
    assert np.max(np.abs(o2 - full_o[41:])) < 1e-13
    # a length-1 sequence returns its own value
    assert np.max(np.abs(full_o[40, 0] - v[40, 0])) < 1e-15


def test_decode_equals_last_prefill_row():
    D, theta, L = 16, 1e4, 90
    q, k, v = _raw_case(L, 4, 2, D, seed=5)
    ref_o, ref_l = oracle.bifocal_attention(q, k, v, [0, L], 20, 7, theta)
    cap = L + 3
    kc = np.zeros((1, cap, 2, D))
    vc = np.zeros((1, cap, 2, D))
    kc[0, :L], vc[0, :L] = k, v
    kc[0, L:] = 1e3  # rows past L must be ignored
    o, l_ = oracle.bifocal_decode(q[L - 1][None], kc, vc, [L], 20, 7, theta)
    assert np.max(np.abs(o[0] - ref_o[L - 1])) < 1e-13
    assert np.max(np.abs(l_[0] - ref_l[:, L - 1])) < 1e-13


# --------------------------------------------------------------------------
# Planted mistakes: each plausible error must make a pin fail
# --------------------------------------------------------------------------


def _brute_force_disagrees():
    L, D, w_pre, w0, theta = 23, 8, 5, 7, 1e4
    q_raw, k_raw, v = _raw_case(L, 1, 1, D, seed=2024)
    pos = np.arange(L)
    # the rotated inputs are made with the unpatched rotation
    qt = _GOOD_ROTATE(q_raw, pos[:, None], theta)
    kt = _GOOD_ROTATE(k_raw, pos[:, None], theta)
    out, _ = oracle.bifocal_attention(qt, kt, v, [0, L], w_pre, w0, theta)
    bo, _ = oracle.brute_force_tiny(q_raw[:, 0].tolist(), k_raw[:, 0].tolist(), v[:, 0].tolist(),
                                    w_pre, w0, theta)
    return np.max(np.abs(out[:, 0] - np.array(bo))) > 1e-6


_GOOD_ROTATE = ob.rope_rotate


def _rotate_wrong_sign(x, m, theta):
    x = np.asarray(x, dtype=np.float64)
    h = x.shape[-1] // 2
    ang = np.asarray(m, dtype=np.float64)[..., None] * ob.rope_inv_freq(x.shape[-1], theta)
    a, b = x[..., :h], x[..., h:]
    return np.concatenate([a * np.cos(ang) + b * np.sin(ang), -a * np.sin(ang) + b * np.cos(ang)], -1)


def _rotate_interleaved_pairs(x, m, theta):
    x = np.asarray(x, dtype=np.float64)
    ang = np.asarray(m, dtype=np.float64)[..., None] * ob.rope_inv_freq(x.shape[-1], theta)
    a, b = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = a * np.cos(ang) - b * np.sin(ang)
    y[..., 1::2] = a * np.sin(ang) + b * np.cos(ang)
    return y


@pytest.mark.parametrize("target,mutant", [
    ("correction_shift", lambda p, G: np.asarray(p) - np.asarray(p) // G),          # sign of delta
    ("position_map", lambda x, G: -(-np.asarray(x, dtype=np.int64) // int(G))),     # ceil, not floor
    ("group_size", lambda L, w: max(1, int(L) // int(w))),                          # floor of L/w
    ("rope_inv_freq", lambda D, th: np.power(float(th), -np.arange(D // 2) / D)),    # exponent k/D
    ("rope_rotate", _rotate_wrong_sign),                                            # rotation sense
    ("rope_rotate", _rotate_interleaved_pairs),                                     # pair layout
])
def test_planted_mistake_is_caught(monkeypatch, target, mutant):
    assert not _brute_force_disagrees()
    monkeypatch.setattr(ob, target, mutant)
    assert _brute_force_disagrees()


def test_planted_window_off_by_one_is_caught():
    # A window that admits w0 + 1 keys must differ from the brute force.
    L, D, w_pre, w0, theta = 23, 8, 5, 7, 1e4
    q_raw, k_raw, v = _raw_case(L, 1, 1, D, seed=2024)
    pos = np.arange(L)
    qt = oracle.rope_rotate(q_raw, pos[:, None], theta)
    kt = oracle.rope_rotate(k_raw, pos[:, None], theta)
    bo, _ = oracle.brute_force_tiny(q_raw[:, 0].tolist(), k_raw[:, 0].tolist(), v[:, 0].tolist(),
                                    w_pre, w0, theta)
    good, _ = oracle.bifocal_attention(qt, kt, v, [0, L], w_pre, w0, theta)
    bad, _ = oracle.bifocal_attention(qt, kt, v, [0, L], w_pre, w0 + 1, theta)
    assert np.max(np.abs(good[:, 0] - np.array(bo))) < 1e-11
    assert np.max(np.abs(bad[:, 0] - np.array(bo))) > 1e-6


# --------------------------------------------------------------------------
# Prefill of new tokens against an existing cache
# --------------------------------------------------------------------------


@pytest.mark.parametrize("L,n,D,w_pre,w0", [(23, 5, 8, 5, 7), (17, 17, 8, 4, 1), (30, 1, 4, 6, 0),
                                            (40, 9, 8, 8, 40), (33, 12, 8, 11, 5)])
def test_chunk_rows_match_pure_python_brute_force(L, n, D, w_pre, w0):
    # queries are the last n positions of an L-token sequence; G = G(L)
    theta = 1e4 if D == 8 else 500.0
    q_raw, k_raw, v = _raw_case(L, 1, 1, D, seed=L * 13 + n)
    qt, kt = _rotated(q_raw, k_raw, theta)
    out, lse = oracle.bifocal_attention_kv(qt[L - n:], kt, v, [0, n], [0, L], w_pre, w0, theta)
    bo, bl = oracle.brute_force_tiny(q_raw[:, 0].tolist(), k_raw[:, 0].tolist(), v[:, 0].tolist(),
                                     w_pre, w0, theta)
    assert np.max(np.abs(out[:, 0] - np.array(bo)[L - n:])) < 1e-11
    assert np.max(np.abs(lse[0] - np.array(bl)[L - n:])) < 1e-11


def test_chunks_of_a_growing_sequence_follow_the_current_length():
    # three chunks appended to one sequence: each chunk's rows equal the full
    # prefill of the prefix that ends with it (G of that prefix), batched varlen
    D, theta, w_pre, w0 = 16, 1e4, 20, 6
    q, k, v = _raw_case(70, 4, 2, D, seed=8)
    bounds = [(0, 25), (25, 41), (41, 70)]
    for a, b in bounds:
        ref_o, ref_l = oracle.bifocal_attention(q[:b], k[:b], v[:b], [0, b], w_pre, w0, theta)
        o, l_ = oracle.bifocal_attention_kv(q[a:b], k[:b], v[:b], [0, b - a], [0, b], w_pre, w0, theta)
        assert np.max(np.abs(o - ref_o[a:b])) < 1e-13
        assert np.max(np.abs(l_ - ref_l[:, a:b])) < 1e-13
    # the same three chunks as one packed batch of three sequences
    cu_q = np.array([0, 25, 41, 70])
    kk = np.concatenate([k[:25], k[:41], k[:70]])
    vv = np.concatenate([v[:25], v[:41], v[:70]])
    cu_k = np.array([0, 25, 66, 136])
    o, _ = oracle.bifocal_attention_kv(q, kk, vv, cu_q, cu_k, w_pre, w0, theta)
    for (a, b) in bounds:
        ref_o, _ = oracle.bifocal_attention(q[:b], k[:b], v[:b], [0, b], w_pre, w0, theta)
        assert np.max(np.abs(o[a:b] - ref_o[a:b])) < 1e-13


def test_one_query_chunk_is_a_decode_step():
    D, theta, L = 16, 1e4, 90
    q, k, v = _raw_case(L, 4, 2, D, seed=21)
    o, l_ = oracle.bifocal_attention_kv(q[L - 1:], k, v, [0, 1], [0, L], 20, 7, theta)
    do, dl = oracle.bifocal_decode(q[L - 1][None], k[None], v[None], [L], 20, 7, theta)
    assert np.max(np.abs(o[0] - do[0])) < 1e-13
    assert np.max(np.abs(l_[:, 0] - dl[0])) < 1e-13


def test_chunk_rejects_more_queries_than_keys():
    q, k, v = _raw_case(5, 1, 1, 4, seed=1)
    with pytest.raises(ValueError):
        oracle.bifocal_attention_kv(q, k[:3], v[:3], [0, 5], [0, 3], 4, 1, 1e4)


# --------------------------------------------------------------------------
# Sliding-window layers of a hybrid model (keys with d >= window masked)
# --------------------------------------------------------------------------


WINDOWED = [  # (L, D, w_pretrained, w0, window)
    (23, 8, 5, 7, 1), (23, 8, 5, 7, 2), (23, 8, 5, 7, 7), (23, 8, 5, 7, 8), (30, 4, 6, 0, 9),
    (33, 8, 11, 5, 17), (17, 8, 4, 1, 16), (19, 8, 4, 3, 40), (40, 8, 8, 12, 25),
]


@pytest.mark.parametrize("L,D,w_pre,w0,window", WINDOWED)
def test_window_rows_match_pure_python_brute_force(L, D, w_pre, w0, window):
    theta = 1e4 if D == 8 else 500.0
    q_raw, k_raw, v = _raw_case(L, 1, 1, D, seed=L * 7 + window)
    qt, kt = _rotated(q_raw, k_raw, theta)
    out, lse = oracle.bifocal_attention(qt, kt, v, [0, L], w_pre, w0, theta, window=window)
    bo, bl = oracle.brute_force_tiny(q_raw[:, 0].tolist(), k_raw[:, 0].tolist(), v[:, 0].tolist(),
                                     w_pre, w0, theta, window=window)
    assert np.max(np.abs(out[:, 0] - np.array(bo))) < 1e-11
    assert np.max(np.abs(lse[0] - np.array(bl))) < 1e-11


@pytest.mark.parametrize("w_pre,w0,window", [(3, 10, 10), (5, 40, 7), (1, 16, 1), (7, 3, 3)])
def test_window_not_wider_than_w0_is_textbook_sliding_window(w_pre, w0, window):
    # every visible pair is local, so G plays no part
    L, D, theta = 64, 16, 1e4
    q, k, v = _raw_case(L, 4, 2, D, seed=window + w0)
    out, lse = oracle.bifocal_attention(q, k, v, [0, L], w_pre, w0, theta, window=window)
    ref_o, ref_l = oracle.causal_rope_attention(q, k, v, window=window)
    assert np.max(np.abs(out - ref_o)) < 1e-13
    assert np.max(np.abs(lse - ref_l)) < 1e-13


def test_window_of_one_returns_each_value():
    # closed form: each query sees only its own key (distance 0, local)
    L, D = 40, 8
    q, k, v = _raw_case(L, 2, 1, D, seed=5)
    out, lse = oracle.bifocal_attention(q, k, v, [0, L], 4, 2, 1e4, window=1)
    for h in range(2):
        assert np.max(np.abs(out[:, h] - v[:, 0])) < 1e-14
        own = np.einsum("id,id->i", q[:, h], k[:, 0]) / math.sqrt(D)
        assert np.max(np.abs(lse[h] - own)) < 1e-13


@pytest.mark.parametrize("window", [60, 61, 1000])
def test_window_covering_the_sequence_changes_nothing(window):
    L, D, theta = 60, 16, 1e4
    q, k, v = _raw_case(L, 4, 1, D, seed=window)
    a, la = oracle.bifocal_attention(q, k, v, [0, L], 16, 5, theta)
    b, lb = oracle.bifocal_attention(q, k, v, [0, L], 16, 5, theta, window=window)
    assert np.array_equal(a, b) and np.array_equal(la, lb)


def test_windowed_decode_equals_last_prefill_row():
    D, theta, L = 16, 1e4, 90
    q, k, v = _raw_case(L, 4, 2, D, seed=31)
    for window in (1, 5, 20, 33, 90):
        po, pl = oracle.bifocal_attention(q, k, v, [0, L], 20, 7, theta, window=window)
        do, dl = oracle.bifocal_decode(q[L - 1][None], k[None], v[None], [L], 20, 7, theta, window=window)
        assert np.max(np.abs(po[L - 1] - do[0])) < 1e-13
        assert np.max(np.abs(pl[:, L - 1] - dl[0])) < 1e-13


def test_planted_sliding_window_off_by_one_is_caught():
    # a window admitting one more key than asked must differ from the brute force
    L, D, w_pre, w0, window, theta = 23, 8, 5, 3, 9, 1e4
    q_raw, k_raw, v = _raw_case(L, 1, 1, D, seed=77)
    qt, kt = _rotated(q_raw, k_raw, theta)
    bo, _ = oracle.brute_force_tiny(q_raw[:, 0].tolist(), k_raw[:, 0].tolist(), v[:, 0].tolist(),
                                    w_pre, w0, theta, window=window)
    good, _ = oracle.bifocal_attention(qt, kt, v, [0, L], w_pre, w0, theta, window=window)
    bad, _ = oracle.bifocal_attention(qt, kt, v, [0, L], w_pre, w0, theta, window=window + 1)
    assert np.max(np.abs(good[:, 0] - np.array(bo))) < 1e-11
    assert np.max(np.abs(bad[:, 0] - np.array(bo))) > 1e-6
