"""Pins for the oracle's binary32 routing recipe (CPU only).

The recipe's exp and log are checked against float64 library routines (an
independent implementation), the log-mean-exp pool against its closed forms and
limits, and the gate against a float64 sigmoid.  Source: HLA summary page,
"Overview" (log-mean-exp pooled routing gates) and "Methodology in Plain English"
(independent sigmoid weights per historical chunk, threshold without
renormalisation).
"""
import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import routing_recipe as rr
from oracle import hla_oracle as ho


def _ulp_err(got, ref):
    ref = np.asarray(ref, np.float64)
    ulp = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)
    return np.abs(np.asarray(got, np.float64) - ref) / ulp


def test_constants_from_mathematics():
    # ln2 head has 16 significant bits: n * LN2_HI is exact for |n| < 256
    bits = np.array([rr.LN2_HI], np.float32).view(np.uint32)[0]
    assert bits & 0xFF == 0
    assert abs(float(rr.LN2_HI) + float(rr.LN2_LO) - math.log(2.0)) < 1e-13
    assert float(rr.EXP_COEF[3]) == float(np.float32(1 / 6))
    assert float(rr.ODD_RECIP[7]) == float(np.float32(1 / 15))


def test_exp32_error_bound():
    x = np.linspace(-85.9, 87.9, 400001, dtype=np.float32)
    err = _ulp_err(rr.exp32(x), np.exp(x.astype(np.float64)))
    assert err.max() <= 1.5
    small = np.linspace(-1e-3, 1e-3, 20001, dtype=np.float32)
    assert _ulp_err(rr.exp32(small), np.exp(small.astype(np.float64))).max() <= 1.5


def test_exp32_special_values():
    assert rr.exp32(np.float32(0.0)) == np.float32(1.0)
    assert np.isinf(rr.exp32(np.float32(88.5)))
    assert rr.exp32(np.float32(-86.5)) == 0.0
    assert rr.exp32(np.float32(-1000.0)) == 0.0
    # exact powers: e^(n ln2) close to 2^n
    for n in (-60, -1, 1, 60):
        assert _ulp_err(rr.exp32(np.float32(n * math.log(2))), math.exp(np.float32(n * math.log(2)))) <= 1.5


def test_log32_error_bound():
    x = np.exp(np.linspace(-60, 60, 400001)).astype(np.float32)
    err = _ulp_err(rr.log32(x), np.log(x.astype(np.float64)))
    assert err.max() <= 2.0
    near1 = (1 + np.linspace(-0.01, 0.01, 20001)).astype(np.float32)
    ref = np.log(near1.astype(np.float64))
    keep = ref != 0
    assert _ulp_err(rr.log32(near1), ref)[keep].max() <= 2.0
    assert rr.log32(np.float32(1.0)) == 0.0
    assert rr.log32(np.float32(1.0 / 64)) == pytest.approx(-math.log(64), rel=2e-7)


def test_lme_single_token_is_identity():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((1, 33)).astype(np.float32)
    for tau in (1.0, 0.5, 3.0):
        r = rr.lme_pool32(x, tau)
        if tau == 1.0:
            assert np.array_equal(r, x[0])
        else:
            np.testing.assert_allclose(r, x[0], rtol=2e-7, atol=1e-7)


def test_lme_identical_tokens_exact():
    rng = np.random.default_rng(1)
    row = rng.standard_normal(17).astype(np.float32)
    x = np.tile(row, (64, 1))
    assert np.array_equal(rr.lme_pool32(x, 1.0), row)


def test_lme_limits_max_and_mean():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 40)).astype(np.float32)
    # tau -> 0+: the pool tends to the max (within tau * log n)
    r = rr.lme_pool32(x, 1e-3)
    assert np.all(np.abs(r - x.max(0)) <= 1e-3 * math.log(64) + 1e-6)
    # large tau: the pool tends to the mean (second-order term var/(2 tau))
    r = rr.lme_pool32(x, 1e3)
    np.testing.assert_allclose(r, x.astype(np.float64).mean(0), atol=2e-3)


def test_lme_matches_float64_definition():
    rng = np.random.default_rng(3)
    for n in (1, 7, 64):
        x = (rng.standard_normal((5, n, 128)) * 3).astype(np.float32)
        got = rr.lme_pool32(x, 1.0)
        ref = rr.lme_pool64(x, 1.0)
        np.testing.assert_allclose(got, ref, rtol=0, atol=4e-6 * np.abs(ref).max())


def test_lme_partial_count():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((64, 8)).astype(np.float32)
    assert np.array_equal(rr.lme_pool32(x, 1.0, n_tokens=5), rr.lme_pool32(x[:5], 1.0))


def test_gate_matches_float64_sigmoid():
    rng = np.random.default_rng(5)
    rq = (rng.standard_normal((50, 128)) * 1.5).astype(np.float32)
    rk = (rng.standard_normal((60, 128)) * 1.5).astype(np.float32)
    g32 = rr.gate_matrix32(rq, rk, 128, -2.0)
    g64 = rr.gate64(rq[:, None, :], rk[None, :, :], 128, -2.0)
    assert np.abs(g32 - g64).max() <= 1e-6
    assert 0.05 < g32.mean() < 0.6  # spread over (0, 1)


def test_gate_saturation():
    one = np.ones((1, 4), np.float32)
    assert rr.gate32(one * 100, one * 100, 4, 0.0) == 1.0
    assert rr.gate32(one * 100, -one * 100, 4, 0.0) == 0.0
    assert rr.gate32(one * 0, one * 0, 4, 0.0) == np.float32(0.5)


def _round_f32(fr: Fraction) -> np.float32:
    """Nearest binary32 to an exact rational, ties to the even significand (brute
    force over the neighbours of a close candidate)."""
    c = np.float32(float(fr))
    cands = [np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))]
    return min(cands, key=lambda v: (abs(Fraction(float(v)) - fr), int(np.array([v]).view(np.uint32)[0]) & 1))


def _fma_exact(a, b, c) -> np.float32:
    return _round_f32(Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c)))


def _midpoint_products(rng, count):
    """Pairs (a, b) of binary32 values whose exact product is a midpoint between two
    neighbouring binary32 values: (2m + 1) 2^k with 2m + 1 split into two factors
    of at most 24 bits."""
    out = []
    while len(out) < count:
        m = int(rng.integers(1 << 23, 1 << 24))
        odd = 2 * m + 1
        f = next((q for q in range(3, 5800, 2) if odd % q == 0), None)
        if f is None or odd // f >= (1 << 24):
            continue
        ka, kb = int(rng.integers(-30, 0)), int(rng.integers(-30, 0))
        out.append((np.float32(math.ldexp(f, ka)), np.float32(math.ldexp(odd // f, kb)), ka + kb))
    return out


def test_fma32_matches_exact_rounding():
    rng = np.random.default_rng(11)
    # random operands over a range of scales
    n = 4000
    a = (rng.standard_normal(n) * np.exp2(rng.integers(-20, 20, n))).astype(np.float32)
    b = (rng.standard_normal(n) * np.exp2(rng.integers(-20, 20, n))).astype(np.float32)
    c = (rng.standard_normal(n) * np.exp2(rng.integers(-40, 40, n))).astype(np.float32)
    got = rr.fma32(a, b, c)
    ref = np.array([_fma_exact(x, y, z) for x, y, z in zip(a, b, c)], np.float32)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    # products that sit exactly on a binary32 midpoint, plus addends far below the
    # float64 resolution of the sum: rounding the float64 sum would tie to even,
    # the single rounding of the exact sum goes the way of the addend's sign
    cases = _midpoint_products(rng, 300)
    a = np.array([x for x, _, _ in cases], np.float32)
    b = np.array([y for _, y, _ in cases], np.float32)
    c = np.array([np.float32(math.ldexp(float(rng.choice([-1.0, 1.0])) * (1 + float(rng.integers(0, 1 << 23)) / 2 ** 23),
                                        k - 40)) for _, _, k in cases], np.float32)
    c[::7] = 0.0  # exact ties: even significand
    got = rr.fma32(a, b, c)
    ref = np.array([_fma_exact(x, y, z) for x, y, z in zip(a, b, c)], np.float32)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    # the float64 sum rounded to binary32 really is wrong on about half of them
    naive = (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)
    assert (naive != ref).sum() >= 60


def test_dot32_is_sequential_fused_sum():
    # with exactly representable partial sums the sequential sum equals the exact one
    a = np.array([1.0, 2.0, 4.0, 8.0], np.float32)
    assert rr.dot32(a, a) == 85.0
    # order matters in binary32: 2^24 + 1 - 2^24 evaluated left to right is 0
    a = np.array([2.0 ** 12, 1.0, 2.0 ** 12], np.float32)
    b = np.array([2.0 ** 12, 1.0, -(2.0 ** 12)], np.float32)
    assert rr.dot32(a, b) == 0.0
    # each step is one fused rounding: (1 + 2^-12)^2 - (1 + 2^-11) = 2^-24 exactly,
    # where a rounded product would give 0
    u = np.float32(1 + 2.0 ** -12)
    a = np.array([-(1 + 2.0 ** -11), u], np.float32)
    b = np.array([1.0, u], np.float32)
    assert rr.dot32(a, b) == np.float32(2.0 ** -24)


def test_gate_matrix_masks_current_and_future():
    rng = np.random.default_rng(6)
    rq = rng.standard_normal((6, 8)).astype(np.float32)
    rk = rng.standard_normal((6, 8)).astype(np.float32)
    G = ho.gate_matrix(rq, rk, 8, 0.0)
    assert np.all(np.triu(G) == 0)
    assert np.all(np.tril(G, -1)[np.tril_indices(6, -1)] > 0)


def test_active_lists_threshold_semantics():
    G = np.zeros((4, 4), np.float32)
    G[3, :3] = [0.049999998, 0.05, 0.9]
    G[2, :2] = [0.01, 0.2]
    act = ho.active_lists(G, 0.05)
    assert [list(a) for a in act] == [[], [], [1], [1, 2]]   # equality is kept
    dense = ho.active_lists(G, 0.0)
    assert [list(a) for a in dense] == [[], [0], [0, 1], [0, 1, 2]]


# ---- window representatives: log-sum-exp over a chunk's windows, then a sigmoid ----

def test_window_gate_matches_float64_definition():
    # the binary32 recipe against sigmoid(log sum_u exp(<rq, rk_u>/sqrt(d)) + b) in fp64
    rng = np.random.default_rng(41)
    d, W = 64, 8
    rq = (rng.standard_normal((200, d)) * 0.8).astype(np.float32)
    rkw = (rng.standard_normal((200, W, d)) * 0.8).astype(np.float32)
    g32 = rr.gate_window32(rq, rkw, d, -2.0)
    g64 = rr.gate_window64(rq, rkw, d, -2.0)
    assert np.abs(g32.astype(np.float64) - g64).max() <= 2e-6


def test_window_gate_of_equal_windows_adds_log_count():
    # W equal representatives: log sum_u exp(t) = t + log W exactly
    rng = np.random.default_rng(42)
    d = 32
    rq = rng.standard_normal(d).astype(np.float32)
    r = rng.standard_normal(d).astype(np.float32)
    for W in (2, 4, 8, 16):
        g = rr.gate_window32(rq, np.tile(r, (W, 1)), d, 0.5)
        t = float(np.dot(rq.astype(np.float64), r.astype(np.float64))) / np.sqrt(d)
        ref = 1.0 / (1.0 + np.exp(-(t + np.log(W) + 0.5)))
        assert abs(float(g) - ref) <= 2e-6


def test_window_gate_follows_the_dominant_window():
    # one window far above the others: the gate tends to the single-window gate of it
    d = 16
    rq = np.zeros(d, np.float32)
    rq[3] = 8.0
    rkw = np.zeros((4, d), np.float32)
    rkw[2, 3] = 8.0                    # score 64 / 4 = 16; the rest score 0
    g = float(rr.gate_window32(rq, rkw, d, -18.0))
    ref = 1.0 / (1.0 + np.exp(-(16.0 + np.log1p(3 * np.exp(-16.0)) - 18.0)))
    assert abs(g - ref) <= 1e-6
    assert abs(g - 1.0 / (1.0 + np.exp(2.0))) <= 1e-5


def test_window_pools_are_per_window_lme():
    rng = np.random.default_rng(43)
    x = rng.standard_normal((3 * 16 + 5, 4)).astype(np.float32)
    r = ho.window_pools(x, 16, 4, 1.0)
    assert r.shape == (3, 4, 4)          # complete chunks only
    for c in range(3):
        for u in range(4):
            seg = x[16 * c + 4 * u:16 * c + 4 * u + 4]
            assert np.array_equal(r[c, u], rr.lme_pool32(seg, 1.0))
