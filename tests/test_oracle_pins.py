"""Pins of the CPU oracle against what the pages and mathematics fix (no GPU needed).

Each test checks the oracle against something other than itself: published known answers,
the pages' worked example, brute force on tiny inputs, an independent naive greedy, Monte
Carlo moments, closed forms and invariants.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


# ------------------------------------------------------------------------------------------
# Philox4x32-10
# ------------------------------------------------------------------------------------------
def test_philox_known_answers():
    rows = _rows("philox4x32_10_kat.txt")
    assert len(rows) == 3
    for r in rows:
        v = [int(x, 16) for x in r]
        out = O.philox(v[0:4], v[4:6])
        assert [int(x) for x in out] == v[6:10]


def test_uniform_statistics():
    # 2^16 draws: mean 1/2, chi-square over 64 bins, round-toward-zero conversion of the word
    n = 1 << 16
    u = np.array([O.uniform(7, 3, 1, i) for i in range(n)], dtype=np.float64)
    assert u.min() >= 0.0 and u.max() < 1.0
    assert abs(u.mean() - 0.5) < 4 * math.sqrt(1 / 12 / n)
    h, _ = np.histogram(u, bins=64, range=(0, 1))
    chi2 = ((h - n / 64) ** 2 / (n / 64)).sum()
    assert chi2 < 63 + 6 * math.sqrt(2 * 63)
    # U * 2^32 is the binary32 value just at or below the generator's word (round toward zero)
    words = []
    for b in range(n // 4):
        words.extend(int(x) for x in O.philox([b, 0, 3, 1], [7, 0]))
    w = np.array(words[:n], dtype=np.float64)
    x = (u * 2.0 ** 32).astype(np.float32)
    assert np.all(x.astype(np.float64) == u * 2.0 ** 32)
    assert np.all(x.astype(np.float64) <= w)
    assert np.all(np.nextafter(x, np.float32(np.inf)).astype(np.float64) > w)
    # distinct workers / steps give distinct streams
    a = [O.uniform(7, 3, 1, i) for i in range(64)]
    b = [O.uniform(7, 3, 2, i) for i in range(64)]
    c = [O.uniform(7, 4, 1, i) for i in range(64)]
    assert a != b and a != c


def test_fexpo_matches_frexp():
    rng = np.random.default_rng(0)
    vals = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.uniform(-40, 38, 2000),
                           [1.0, 2.0, 0.5, 1e-45, 1.4e-45, 3e-39, 1.1754942e-38, 1.1754944e-38, 3.4e38]])
    for v in np.abs(vals.astype(np.float32)):
        if v == 0:
            continue
        m, e = math.frexp(float(v))
        assert O.fexpo(float(v)) == e - 1


# ------------------------------------------------------------------------------------------
# Stochastic rounding: the pages' worked example and Monte Carlo moments
# ------------------------------------------------------------------------------------------
def _mc(cfg, v, steps):
    qs = np.stack([O.encode_bucket(cfg, 0, t, 0, v)[1] for t in range(steps)]).astype(np.float64)
    return qs


def test_worked_example_point_seven():
    (val, lo, hi, p_up), = [[float(x) for x in r] for r in _rows("stochastic_rounding_example.txt")]
    d = 512
    v = np.full(d, val, dtype=np.float32)
    v[0], v[1] = lo, hi          # ORQ-2 levels are the bucket's min and max: exactly {0, 1}
    cfg = O.Config(O.ORQ, 2, d, 1, 1, 0.0, 42, d)
    _, _, table = O.encode_bucket(cfg, 0, 0, 0, v)
    assert list(table) == [lo, hi]
    steps = 200                   # 510 draws per step: 102,000 draws
    qs = _mc(cfg, v, steps)[:, 2:]
    frac_up = (qs == hi).mean()
    assert set(np.unique(qs)) <= {lo, hi}
    sigma = math.sqrt(p_up * (1 - p_up) / qs.size)
    assert abs(frac_up - p_up) < 3 * sigma
    # QSGD-3 with m = 1 has levels {-1, 0, 1}: 0.7 lies between 0 and 1 as well
    v2 = np.full(d, val, dtype=np.float32)
    v2[0] = -1.0
    cfgq = O.Config(O.QSGD, 3, d, 1, 1, 0.0, 42, d)
    qq = _mc(cfgq, v2, steps)[:, 1:]
    assert set(np.unique(qq)) <= {0.0, 1.0}
    assert abs((qq == 1.0).mean() - p_up) < 3 * math.sqrt(0.21 / qq.size)


def _bracket_moments(levels, u):
    """(lower, upper) adjacent levels of each value in an ascending level list."""
    lv = np.asarray(levels, dtype=np.float64)
    k = np.clip(np.searchsorted(lv, u, side="right") - 1, 0, len(lv) - 2)
    return lv[k], lv[k + 1]


@pytest.mark.parametrize("scheme,levels", [(O.ORQ, 3), (O.ORQ, 5), (O.ORQ, 9), (O.QSGD, 5),
                                           (O.TERNGRAD, 3), (O.QSGD, 9)])
def test_unbiased_and_variance_monte_carlo(scheme, levels):
    rng = np.random.default_rng(scheme * 10 + levels)
    d = 128
    v = (rng.laplace(0, 1e-3, d)).astype(np.float32)
    cfg = O.Config(scheme, levels, d, 1, 1, 0.0, 99, d)
    steps = 1000                  # 1000 draws per element, 128,000 draws
    qs = _mc(cfg, v, steps)
    _, _, table = O.encode_bucket(cfg, 0, 0, 0, v)
    if scheme in (O.QSGD, O.TERNGRAD):
        m = float(table[0])
        lv = [m * (2 * k - (levels - 1)) / (levels - 1) for k in range(levels)]
    else:
        lv = [float(t) for t in table]
    assert all(lv[i] <= lv[i + 1] for i in range(len(lv) - 1))
    u = v.astype(np.float64)
    a, b = _bracket_moments(lv, u)
    var = (b - u) * (u - a)
    # every output is a level and lies in the fitted range
    assert qs.min() >= lv[0] and qs.max() <= lv[-1]
    assert np.isin(qs.astype(np.float32), np.asarray(lv, dtype=np.float32)).all()
    mean = qs.mean(axis=0)
    se = np.sqrt(np.maximum(var, 1e-30) / steps)
    z = (mean - u) / se
    ok = var > 0
    assert np.abs(z[ok]).max() < 5.5
    assert 0.75 < np.mean(z[ok] ** 2) < 1.25
    # deterministic where the value sits on a level
    assert np.allclose(mean[~ok], u[~ok], rtol=0, atol=1e-6 * abs(lv[-1] - lv[0]))
    # expected variance sum (b-x)(x-a) against the empirical one
    emp = qs.var(axis=0).sum()
    assert abs(emp - var.sum()) < 0.1 * var.sum()


# ------------------------------------------------------------------------------------------
# ORQ greedy
# ------------------------------------------------------------------------------------------
def _naive_orq(u, s):
    """Independent greedy on the raw values in float64 (no fixed point, no prefix sums)."""
    x = np.asarray(u, dtype=np.float64)
    mn, mx = x.min(), x.max()
    grid = mn + np.arange(64) * (mx - mn) / 63.0
    grid[63] = mx

    def total(lvset):
        a, b = _bracket_moments(grid[sorted(lvset)], x)
        return float(np.sum((b - x) * (x - a)))

    lv = [0, 63]
    for _ in range(s - 2):
        best = None
        for c in range(1, 63):
            if c in lv:
                continue
            t = total(lv + [c])
            if best is None or t < best[0]:
                best = (t, c)
        lv.append(best[1])
    return sorted(lv), total(lv), total


@pytest.mark.parametrize("s", [2, 3, 5, 9])
def test_orq_matches_naive_greedy(s):
    """The fixed-point greedy (positions with 16 fraction bits per grid cell, exact integer
    objective) against an independent greedy on the raw values in float64.  Every pick must be
    as good as the real-valued one to 1e-9 relative; on normal and Laplace buckets the picks
    must be the same levels.  (Measured on 300 buckets of d = 512 per workload distribution and
    s = 3, 5, 9: the picks differ only on Student-t buckets with outliers, where candidates tie
    exactly -- the real-valued variances differ by at most 1.1e-13 relative.)"""
    rng = np.random.default_rng(s)
    trials = 12
    for t in range(trials):
        n = int(rng.integers(40, 300))
        dist = t % 3
        if dist == 0:
            u = rng.standard_normal(n)
        elif dist == 1:
            u = rng.laplace(0, 1, n)
        else:
            u = rng.standard_t(3, n)
        u = (u * 1e-3).astype(np.float32)
        var_fixed, idx = O.orq_select(u, s)
        lv, tot, total = _naive_orq(u, s)
        assert sorted(idx.tolist()) == idx.tolist()
        assert idx[0] == 0 and idx[-1] == 63
        mine = total(list(idx))
        assert mine <= tot * (1 + 1e-9) + 1e-30
        if dist < 2:
            assert list(idx) == lv, (t, list(idx), lv)


def test_orq_greedy_nested_and_monotone():
    rng = np.random.default_rng(5)
    u = (rng.standard_normal(512) * 1e-3).astype(np.float32)
    prev_idx, prev_var = None, None
    for s in range(2, 12):
        var, idx = O.orq_select(u, s)
        if prev_idx is not None:
            assert set(prev_idx.tolist()) <= set(idx.tolist())
            assert var <= prev_var
        prev_idx, prev_var = idx, var


def test_orq_three_point_special_case():
    # values only on grid points {g_0, g_k, g_63}: ORQ-3 picks k, zero variance, no randomness
    d = 256
    k = 23
    lo, hi = -0.5, 1.0
    rng = np.random.default_rng(3)
    ok, grid = O.grid(np.array([lo, hi], dtype=np.float32))
    assert ok
    v = grid[rng.choice([0, k, 63], size=d)].astype(np.float32)
    v[0], v[1], v[2] = grid[0], grid[k], grid[63]
    var, idx = O.orq_select(v, 3)
    assert idx.tolist() == [0, k, 63]
    assert var == 0.0
    cfg = O.Config(O.ORQ, 3, d, 1, 1, 0.0, 5, d)
    for step in range(4):
        code, q, table = O.encode_bucket(cfg, 0, step, 0, v)
        assert np.array_equal(q, v)


def test_orq2_is_min_max():
    rng = np.random.default_rng(8)
    u = (rng.standard_normal(300)).astype(np.float32)
    cfg = O.Config(O.ORQ, 2, 512, 1, 1, 0.0, 1, 300)
    _, q, table = O.encode_bucket(cfg, 0, 0, 0, u)
    assert table[0] == u.min() and table[1] == u.max()
    assert set(np.unique(q)) <= {u.min(), u.max()}


def test_orq_constant_bucket():
    cfg = O.Config(O.ORQ, 5, 128, 1, 1, 0.0, 1, 128)
    v = np.full(128, 0.25, dtype=np.float32)
    code, q, table = O.encode_bucket(cfg, 0, 0, 0, v)
    assert (code == 0).all() and (q == 0.25).all() and (table == 0.25).all()


# ------------------------------------------------------------------------------------------
# BinGrad-b: brute force over every threshold (exact rational arithmetic)
# ------------------------------------------------------------------------------------------
def _sse_split(vals, k):
    left, right = vals[:k], vals[k:]
    fl = [Fraction(float(x)) for x in left]
    fr = [Fraction(float(x)) for x in right]
    ml = sum(fl) / len(fl)
    mr = sum(fr) / len(fr)
    return sum((x - ml) ** 2 for x in fl) + sum((x - mr) ** 2 for x in fr)


def test_bingrad_b_brute_force():
    rng = np.random.default_rng(11)
    for t in range(60):
        n = int(rng.integers(2, 17))
        if t % 4 == 0:
            u = rng.choice([-1.0, 0.5, 2.0], size=n)      # many ties
        else:
            u = rng.standard_normal(n) * 10.0 ** rng.uniform(-5, 1)
        u = u.astype(np.float32)
        a, b, thr, split = O.bingrad_b_fit(u)
        srt = np.sort(u)
        cands = [k for k in range(1, n) if srt[k - 1] < srt[k]]
        if not cands:
            assert split == 0 and a == b == srt[0]
            continue
        best = min(_sse_split(srt, k) for k in cands)
        mine = _sse_split(srt, split)
        assert srt[split - 1] < srt[split] and thr == srt[split]
        assert float(mine) <= float(best) * (1 + 1e-9) + 1e-300
        # levels are the side means (rounded to binary32)
        ml = float(sum(Fraction(float(x)) for x in srt[:split]) / split)
        mr = float(sum(Fraction(float(x)) for x in srt[split:]) / (n - split))
        assert abs(a - ml) <= 2e-7 * max(abs(ml), 1e-30) and abs(b - mr) <= 2e-7 * max(abs(mr), 1e-30)
        # Lloyd condition: every value is at least as near its own level
        for x in srt[:split]:
            assert abs(float(x) - ml) <= abs(float(x) - mr) * (1 + 1e-6) + 1e-12 * abs(mr - ml)
        for x in srt[split:]:
            assert abs(float(x) - mr) <= abs(float(x) - ml) * (1 + 1e-6) + 1e-12 * abs(mr - ml)


def test_bingrad_b_codes_deterministic():
    rng = np.random.default_rng(12)
    v = (rng.standard_normal(512) * 1e-3).astype(np.float32)
    cfg = O.Config(O.BINGRAD_B, 2, 512, 1, 1, 0.0, 3, 512)
    c0, q0, t0 = O.encode_bucket(cfg, 0, 0, 0, v)
    c1, q1, t1 = O.encode_bucket(cfg, 0, 7, 0, v)
    assert np.array_equal(c0, c1) and np.array_equal(q0, q1)
    a, b, thr, _ = O.bingrad_b_fit(v)
    assert np.array_equal(c0, (v >= thr).astype(np.uint8))


# ------------------------------------------------------------------------------------------
# BinGrad-pb: the properties [P2] states (a wider range and less bias than BinGrad-b, a larger
# error), and brute force over the admissible grid pairs
# ------------------------------------------------------------------------------------------
def _pb_error(x, a, b):
    x = np.asarray(x, dtype=np.float64)
    e = np.where(x < a, (a - x) ** 2, np.where(x >= b, (x - b) ** 2, (b - x) * (x - a)))
    return float(e.sum())


def _grid32(u):
    """The 64-point grid in binary32: min + j * ((max - min) / 63), the last point max."""
    mn, mx = np.float32(u.min()), np.float32(u.max())
    step = np.float32(mx - mn) / np.float32(63.0)
    g = np.array([np.float32(mn + np.float32(j) * step) for j in range(64)], dtype=np.float32)
    g[63] = mx
    return g


def _pb_buckets(seed, count, n=512):
    rng = np.random.default_rng(seed)
    draws = [rng.standard_normal, lambda k: rng.laplace(0, 1, k), lambda k: rng.standard_t(3, k),
             lambda k: rng.uniform(-1, 1, k)]
    return [(draws[t % 4](n) * 1e-3).astype(np.float32) for t in range(count)]


def test_bingrad_pb_brute_force():
    """The pair minimises the expected squared error over every grid pair at least as wide as
    BinGrad-b's levels (brute force on the values in binary64)."""
    rng = np.random.default_rng(13)
    for t in range(24):
        n = int(rng.integers(8, 160))
        u = (rng.standard_t(3, n) if t % 2 else rng.laplace(0, 1, n)) * 1e-3
        u = u.astype(np.float32)
        A, B, ga, gb = O.bingrad_pb_fit(u)
        a_b, b_b, _, _ = O.bingrad_b_fit(u)
        grid = _grid32(u)
        x = u.astype(np.float64)
        ok = [(i, j) for i in range(63) for j in range(i + 1, 64)
              if (grid[i] <= a_b or i == 0) and (grid[j] >= b_b or j == 63)]
        best = min(_pb_error(x, float(grid[i]), float(grid[j])) for i, j in ok)
        assert (A, B) in ok
        assert (ga, gb) == (grid[A], grid[B])
        assert _pb_error(x, ga, gb) <= best * (1 + 1e-4) + 1e-30


# Integer buckets on which the best admissible pair lies inside the admissible corner (found
# by a search over random integer buckets); the expected pairs are computed below.
_PB_INNER = [[0, 2, 3, 30, 52, 53, 63], [0, 1, 29, 63], [0, 31, 50, 63], [0, 7, 14, 35, 61, 61, 63],
             [0, 34, 62, 63], [0, 33, 57, 63], [0, 3, 30, 48, 63], [0, 1, 31, 57, 62, 63], [0, 11, 32, 63],
             [0, 1, 29, 62, 62, 63], [0, 11, 13, 33, 56, 62, 63], [0, 2, 29, 59, 61, 63], [0, 12, 12, 33, 59, 63],
             [0, 2, 9, 30, 57, 59, 63], [0, 3, 30, 56, 58, 63], [0, 11, 33, 57, 61, 63], [0, 1, 5, 32, 62, 63],
             [0, 7, 31, 63], [0, 2, 4, 33, 60, 63], [0, 1, 33, 60, 63], [0, 1, 1, 5, 28, 53, 63],
             [0, 33, 61, 63], [0, 10, 33, 60, 63], [0, 1, 3, 33, 62, 63], [0, 15, 33, 61, 63],
             [0, 2, 30, 61, 63], [0, 5, 32, 58, 63], [0, 1, 1, 29, 63], [0, 32, 59, 63], [0, 15, 33, 63],
             [0, 8, 8, 34, 62, 63], [0, 4, 6, 30, 51, 53, 57, 59, 63], [0, 6, 33, 62, 63], [0, 4, 29, 63],
             [0, 4, 30, 60, 63], [0, 31, 52, 63], [0, 3, 32, 59, 63], [0, 11, 13, 32, 63]]


def test_bingrad_pb_exact_on_the_integer_grid():
    """Small buckets of integers with minimum 0 and maximum 63: the grid is 0..63 exactly and the
    positions are exact, so the pair must equal an exact-integer brute force over the
    admissible pairs (ties to the smallest (A, B))."""
    from fractions import Fraction
    rng = np.random.default_rng(16)
    cases = _PB_INNER + [[0, 63] + rng.integers(1, 63, int(rng.integers(1, 7))).tolist() for _ in range(150)]
    inner = 0
    for x in cases:
        xs = sorted(x)
        n = len(xs)
        best = None
        for k in range(1, n):  # BinGrad-b's split, exactly
            if xs[k - 1] < xs[k]:
                J = Fraction(sum(xs[:k])) ** 2 / k + Fraction(sum(xs[k:])) ** 2 / (n - k)
                if best is None or J > best[0]:
                    best = (J, k)
        k = best[1]
        a_b, b_b = Fraction(sum(xs[:k]), k), Fraction(sum(xs[k:]), n - k)
        amax = max(j for j in range(64) if j <= a_b)
        bmin = min(j for j in range(64) if j >= b_b)

        def err(A, B):
            return sum((A - v) ** 2 if v < A else (v - B) ** 2 if v >= B else (B - v) * (v - A) for v in x)
        pair = min(((err(A, B), A, B) for A in range(amax + 1) for B in range(max(A + 1, bmin), 64)))
        inner += (pair[1], pair[2]) != (amax, bmin)
        A, B, ga, gb = O.bingrad_pb_fit(np.array(x, dtype=np.float32))
        assert (A, B) == (pair[1], pair[2]), (x, (A, B), pair)
        assert (ga, gb) == (float(A), float(B))
    assert inner >= len(_PB_INNER)


def test_bingrad_pb_wider_range_than_b():
    """[P2] Proposed method: BinGrad-pb reduces bias with a wider range than BinGrad-b."""
    for u in _pb_buckets(31, 200):
        a, b, _, _ = O.bingrad_b_fit(u)
        _, _, ga, gb = O.bingrad_pb_fit(u)
        assert ga <= a and gb >= b
        assert gb - ga >= b - a


def test_bingrad_pb_less_bias_than_b():
    """[P2] Proposed method: BinGrad-pb reduces bias.  Its expected value differs from a value only
    where the value is clamped, and by less than BinGrad-b's deterministic error there."""
    for u in _pb_buckets(32, 120):
        a, b, thr, _ = O.bingrad_b_fit(u)
        _, _, ga, gb = O.bingrad_pb_fit(u)
        x = u.astype(np.float64)
        bias_pb = np.where(x < ga, ga - x, np.where(x > gb, x - gb, 0.0))
        err_b = np.abs(np.where(x >= thr, b, a) - x)
        assert np.all(bias_pb <= err_b * (1 + 1e-6) + 1e-12)
        assert bias_pb.sum() < err_b.sum()


def test_bingrad_b_error_below_pb():
    """[P2] Key findings: BinGrad-b's quantization error is lower than BinGrad-pb's."""
    rng = np.random.default_rng(14)
    for t in range(10):
        n = 128
        u = [rng.standard_normal(n), rng.laplace(0, 1, n), rng.standard_t(3, n)][t % 3]
        u = (u * 1e-3).astype(np.float32)
        a, b, thr, split = O.bingrad_b_fit(u)
        x = u.astype(np.float64)
        sse_b = float(np.sum(np.where(x >= thr, (x - b) ** 2, (x - a) ** 2)))
        _, _, ga, gb = O.bingrad_pb_fit(u)
        assert sse_b <= _pb_error(x, ga, gb) * (1 + 1e-6)


def test_bingrad_pb_unbiased_inside_range():
    rng = np.random.default_rng(15)
    d = 128
    v = (rng.standard_normal(d) * 1e-3).astype(np.float32)
    cfg = O.Config(O.BINGRAD_PB, 2, d, 1, 1, 0.0, 17, d)
    qs = _mc(cfg, v, 600)
    _, _, table = O.encode_bucket(cfg, 0, 0, 0, v)
    a, b = float(table[0]), float(table[1])
    x = v.astype(np.float64)
    inside = (x > a) & (x < b)
    assert inside.sum() > 10
    mean = qs.mean(axis=0)
    se = np.sqrt(np.maximum((b - x) * (x - a), 0) / qs.shape[0])
    z = (mean[inside] - x[inside]) / se[inside]
    assert np.abs(z).max() < 5.5
    assert np.all(mean[x <= a] == a) and np.all(mean[x >= b] == b)


# ------------------------------------------------------------------------------------------
# QSGD / TernGrad closed forms
# ------------------------------------------------------------------------------------------
def test_qsgd_levels_and_exact_points():
    d = 128
    for s in (3, 5, 9):
        m = 0.75
        levels = [m * (2 * k - (s - 1)) / (s - 1) for k in range(s)]
        v = np.array([levels[i % s] for i in range(d)], dtype=np.float32)
        cfg = O.Config(O.QSGD, s, d, 1, 1, 0.0, 2, d)
        for step in range(3):
            code, q, table = O.encode_bucket(cfg, 0, step, 0, v)
            assert table[0] == np.float32(m)
            assert np.array_equal(q, v)                 # values on levels are exact
            assert np.array_equal(code, np.arange(d) % s)


def test_terngrad_is_qsgd3():
    rng = np.random.default_rng(16)
    v = (rng.standard_normal(512) * 1e-3).astype(np.float32)
    a = O.encode_bucket(O.Config(O.TERNGRAD, 3, 512, 1, 1, 0.0, 4, 512), 0, 2, 3, v)
    b = O.encode_bucket(O.Config(O.QSGD, 3, 512, 1, 1, 0.0, 4, 512), 0, 2, 3, v)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    m = float(np.abs(v).max())
    assert set(np.unique(a[1]).tolist()) <= {-m, 0.0, m}


def test_zero_bucket_all_schemes():
    v = np.zeros(256, dtype=np.float32)
    for sch, s in [(O.QSGD, 5), (O.TERNGRAD, 3), (O.BINGRAD_B, 2), (O.BINGRAD_PB, 2), (O.ORQ, 5)]:
        code, q, table = O.encode_bucket(O.Config(sch, s, 256, 1, 1, 0.0, 1, 256), 0, 0, 0, v)
        assert (q == 0).all()


# ------------------------------------------------------------------------------------------
# Clipping, packing, error feedback, aggregation
# ------------------------------------------------------------------------------------------
def test_clip_threshold_is_c_sigma():
    rng = np.random.default_rng(17)
    for t in range(20):
        n = int(rng.integers(2, 600))
        v = (rng.standard_t(3, n) * 10.0 ** rng.uniform(-6, 0)).astype(np.float32)
        T = O.clip_threshold(v, 2.5)
        sigma = v.astype(np.float64).std()
        assert abs(T - 2.5 * sigma) <= 2e-5 * 2.5 * sigma + 1e-30
    assert O.clip_threshold(np.zeros(10, dtype=np.float32), 2.5) == 0.0
    v = (rng.standard_normal(512) * 1e-3).astype(np.float32)
    v[5] = 1.0
    cfg = O.Config(O.ORQ, 3, 512, 1, 1, 2.5, 1, 512)
    _, q, table = O.encode_bucket(cfg, 0, 0, 0, v)
    T = O.clip_threshold(v, 2.5)
    assert table[-1] <= T and table[0] >= -T and np.abs(q).max() <= T


@pytest.mark.parametrize("levels", [2, 3, 4, 5, 9, 16, 255])
def test_pack_roundtrip(levels):
    rng = np.random.default_rng(levels)
    for d in (128, 512, 2048):
        for n in (d, d - 1, 40, 1):
            cfg = O.Config(O.ORQ, levels, d, 1, 1, 0.0, 0, n)
            code = rng.integers(0, levels, n).astype(np.uint8)
            words = O.pack_bucket(cfg, code)
            assert words.size == d * O.bits(levels) // 32
            assert np.array_equal(O.unpack_bucket(cfg, words, n), code)
            ones = sum(bin(int(w)).count("1") for w in words)
            assert ones == sum(bin(int(c)).count("1") for c in code)
            if n < d:  # padding codes are zero
                assert np.array_equal(O.unpack_bucket(cfg, words, d)[n:], np.zeros(d - n, np.uint8))


@pytest.mark.parametrize("levels", [2, 3, 5, 9, 16, 255])
def test_pack_is_dense_little_endian(levels):
    """Packing layout: element e's code is bits b*e .. b*e+b-1 of the bucket's little-endian
    bit string (here built as one Python integer, independently of the C loop); 255 levels
    give the byte codes of INT8."""
    rng = np.random.default_rng(100 + levels)
    b = O.bits(levels)
    for d, n in ((128, 128), (512, 512), (512, 301), (1024, 1000)):
        cfg = O.Config(O.ORQ, levels, d, 1, 1, 0.0, 0, n)
        code = rng.integers(0, levels, n).astype(np.uint8)
        stream = 0
        for e in range(n):
            stream |= int(code[e]) << (b * e)
        expect = np.array([(stream >> (32 * k)) & 0xffffffff for k in range(d * b // 32)], dtype=np.uint32)
        assert np.array_equal(O.pack_bucket(cfg, code), expect)


def test_error_feedback_telescopes():
    """[P3] error feedback: nothing is lost, only delayed: sum_t Q_t = sum_t g_t + r_0 - r_T."""
    rng = np.random.default_rng(18)
    n, d, T = 1000, 128, 6
    cfg = O.Config(O.ORQ, 3, d, 1, 1, 0.0, 9, n)
    r = np.zeros(n, dtype=np.float32)
    r0 = r.copy()
    gsum = np.zeros(n)
    qsum = np.zeros(n)
    for t in range(T):
        g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
        gsum += g
        rin = r.copy()
        msg = O.encode(cfg, 0, t, g, r)
        avg = O.decode_accumulate(O.Config(O.ORQ, 3, d, 1, 1, 0.0, 9, n), [msg])
        qsum += avg
        assert np.allclose(avg, (g + rin) - r, rtol=0, atol=1e-9)
    assert np.allclose(qsum, gsum + r0 - r, rtol=0, atol=5e-9)


def test_fused_equals_encode_then_decode():
    rng = np.random.default_rng(19)
    n, d, W = 1000, 128, 3
    for sch, s in [(O.ORQ, 5), (O.QSGD, 5), (O.BINGRAD_B, 2), (O.BINGRAD_PB, 2)]:
        cfg = O.Config(sch, s, d, W, 1, 0.0, 21, n)
        gs = [(rng.standard_normal(n) * 1e-3).astype(np.float32) for _ in range(W)]
        rs = [(rng.standard_normal(n) * 1e-5).astype(np.float32) for _ in range(W)]
        rs2 = [r.copy() for r in rs]
        avg, msgs = O.fused_step(cfg, 4, gs, rs)
        msgs2 = [O.encode(cfg, w, 4, gs[w], rs2[w]) for w in range(W)]
        avg2 = O.decode_accumulate(cfg, msgs2)
        assert all(np.array_equal(a, b) for a, b in zip(msgs, msgs2))
        assert all(np.array_equal(a, b) for a, b in zip(rs, rs2))
        assert np.array_equal(avg, avg2)
        # the average is the mean of the workers' dequantized values, read back from the
        # messages bucket by bucket
        _, coff, loff = O.message_layout(cfg)
        L = O.table_len(sch, s)
        wpb = d * O.bits(s) // 32
        deq = np.zeros((W, n))
        for w in range(W):
            words = msgs[w][coff:loff].view(np.uint32)
            tables = msgs[w][loff:].view(np.float32)
            for bk in range(O.num_buckets(cfg)):
                nb_ = min(d, n - bk * d)
                codes = O.unpack_bucket(cfg, words[bk * wpb:(bk + 1) * wpb], nb_)
                tab = tables[bk * L:(bk + 1) * L]
                deq[w, bk * d:bk * d + nb_] = [O.dequant(cfg, tab, int(c)) for c in codes]
        assert np.allclose(avg, deq.mean(axis=0), rtol=1e-6, atol=1e-12)


def test_message_sizes_and_compression():
    rows = _rows("compression_ratios.txt")
    for s, bits, ratio in rows[:2]:
        assert round(32 / math.log2(int(s)), 1) == float(ratio)
    assert O.bits(3) == 2 and O.bits(5) == 3 and O.bits(9) == 4 and O.bits(2) == 1
    # the glossary's TernGrad (16x) and SignSGD (32x) figures are the codes alone: 2 and 1 bits
    for s, bits, ratio in rows[3:5]:
        assert O.bits(int(s)) == int(bits) and 32 // O.bits(int(s)) == int(ratio)
    assert O.table_len(O.SIGNSGD, 2) == 2 and O.table_len(O.QSGD_NEAREST, 3) == 1
    n = 512 * 1000
    cfg = O.Config(O.ORQ, 5, 512, 1, 1, 0.0, 0, n)
    nbytes, coff, loff = O.message_layout(cfg)
    assert loff == n * 3 // 8 and nbytes == loff + 1000 * 5 * 4
    assert abs(32 * n / (8 * nbytes) - 32 / (3 + 5 * 32 / 512)) < 1e-9


def test_tie_rules():
    # Only the two end values: every candidate leaves the variance at 0, so ORQ must take the
    # smallest unused grid indices, one per round.
    u = np.array([-1.0, 2.0] * 50, dtype=np.float32)
    assert O.orq_select(u, 3)[1].tolist() == [0, 1, 63]
    assert O.orq_select(u, 5)[1].tolist() == [0, 1, 2, 3, 63]
    # {-1, 0, 1}: the splits after the first and after the second value have equal SSE (1/2);
    # the smaller split wins.
    a, b, thr, split = O.bingrad_b_fit(np.array([1.0, -1.0, 0.0], dtype=np.float32))
    assert (split, thr, a, b) == (1, 0.0, -1.0, 0.5)
    # BinGrad-pb on the integer grid 0..63 (min 0, max 63) for {0, 1, 30, 63}: BinGrad-b's levels
    # are 1/2 and 93/2, so A <= 0 and B >= 47; the pairs (0, 47) and (0, 48) both give the least
    # expected squared error, 812 (0 + 46 + 17 * 30 + 16^2 = 0 + 47 + 18 * 30 + 15^2); the
    # smaller wins.
    A, B, ga, gb = O.bingrad_pb_fit(np.array([0.0, 1.0, 30.0, 63.0], dtype=np.float32))
    assert (A, B, ga, gb) == (0, 47, 0.0, 47.0)


# ------------------------------------------------------------------------------------------
# Quantization error (expected and realised), the quantity the bucket sweep reports
# ------------------------------------------------------------------------------------------
def test_quant_error_matches_brackets_and_monte_carlo():
    rng = np.random.default_rng(21)
    n, d = 3 * 128 + 50, 128
    g = (rng.laplace(0, 1e-3, n)).astype(np.float32)
    for sch, s in [(O.ORQ, 5), (O.ORQ, 3), (O.QSGD, 5), (O.TERNGRAD, 3)]:
        cfg = O.Config(sch, s, d, 1, 0, 0.0, 8, n)
        e, uu, qq = O.quant_error(cfg, 0, 0, g)
        assert abs(uu - float(np.sum(g.astype(np.float64) ** 2))) <= 1e-12 * uu
        # expected error = sum (b-u)(u-a) over the brackets of the message's levels
        msg = O.encode(cfg, 0, 0, g)
        _, _, loff = O.message_layout(cfg)
        L = O.table_len(sch, s)
        tabs = msg[loff:].view(np.float32)
        ref = 0.0
        for bk in range(O.num_buckets(cfg)):
            x = g[bk * d:(bk + 1) * d].astype(np.float64)
            t = tabs[bk * L:(bk + 1) * L]
            lv = [float(t[0]) * (2 * k - (s - 1)) / (s - 1) for k in range(s)] if sch in (O.QSGD, O.TERNGRAD) \
                else [float(v) for v in t]
            a, b = _bracket_moments(lv, x)
            ref += float(np.sum(np.maximum((b - x) * (x - a), 0.0)))
        assert abs(e - ref) <= 1e-6 * ref
        # the realised error averages to the expected one
        reps = np.array([O.quant_error(cfg, 0, t, g)[2] for t in range(300)])
        assert abs(reps.mean() - e) < 5 * reps.std() / np.sqrt(len(reps)) + 1e-3 * e


def test_quant_error_deterministic_schemes():
    rng = np.random.default_rng(22)
    n, d = 600, 128
    g = (rng.standard_t(3, n) * 1e-3).astype(np.float32)
    cfg = O.Config(O.BINGRAD_B, 2, d, 1, 0, 0.0, 1, n)
    e, uu, qq = O.quant_error(cfg, 0, 0, g)
    assert e == qq
    sse = 0.0
    for bk in range(O.num_buckets(cfg)):
        x = g[bk * d:(bk + 1) * d]
        a, b, thr, split = O.bingrad_b_fit(x)
        xx = x.astype(np.float64)
        sse += float(np.sum(np.where(xx >= thr, (xx - b) ** 2, (xx - a) ** 2)))
    assert abs(e - sse) <= 1e-9 * sse
    cfg = O.Config(O.BINGRAD_PB, 2, d, 1, 0, 0.0, 1, n)
    e, uu, qq = O.quant_error(cfg, 0, 0, g)
    ref = 0.0
    for bk in range(O.num_buckets(cfg)):
        x = g[bk * d:(bk + 1) * d]
        _, _, ga, gb = O.bingrad_pb_fit(x)
        ref += _pb_error(x, ga, gb)
    # the clamp regions are decided on 16-bit grid positions, the formula here on values:
    # elements within a position step of a level may fall on either side
    assert abs(e - ref) <= 1e-6 * ref


# ------------------------------------------------------------------------------------------
# Base-s packing of the codes ([P2] "Key findings": compression ratios 20.2 for 3 levels and
# 10.1 for 9 levels, i.e. 32 / log2(s) bits)
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("levels", [3, 5, 9])
def test_entropy_groups_near_log2(levels):
    """g codes of s levels fit B bits (s^g <= 2^B, B minimal), and B/g is within 1 % of the
    entropy bound log2(s): the ratio 32*g/B is within 1 % of the pages' 32 / log2(s)."""
    g, B = O.entropy_groups(levels)
    assert levels ** g <= 2 ** B < 2 * levels ** g
    assert abs(B / g - math.log2(levels)) / math.log2(levels) < 0.01
    printed = {int(r[0]): float(r[2]) for r in _rows("compression_ratios.txt")[:2]}  # 3 -> 20.2, 9 -> 10.1
    if levels in printed:
        assert abs(32 * g / B - printed[levels]) / printed[levels] < 0.01
    assert O.entropy_groups(4) is None and O.entropy_groups(2) is None and O.entropy_groups(16) is None


@pytest.mark.parametrize("levels", [3, 5, 9])
def test_entropy_sizes(levels):
    """Words per bucket ceil(ceil(d/g)*B/32) and the layout's 16-byte-aligned regions."""
    g, B = O.entropy_groups(levels)
    for d, n in ((128, 1000), (512, 512 * 3 + 7), (2048, 2048)):
        cfg = O.Config(O.ORQ, levels, d, 1, 1, 0.0, 0, n)
        ew = -(-(-(-d // g)) * B // 32)
        assert O.entropy_words(cfg) == ew
        nb = -(-n // d)
        tl = O.table_len(O.ORQ, levels)
        nbytes, coff, loff = O.entropy_layout(cfg)
        assert coff == 0 and loff == -(-nb * ew * 4 // 16) * 16
        assert nbytes == loff + -(-nb * tl * 4 // 16) * 16
    # d = 512: 26, 38 and 52 words against 32, 48 and 64 of the dense message
    assert O.entropy_words(O.Config(O.ORQ, levels, 512, 1, 1, 0.0, 0, 512)) == {3: 26, 5: 38, 9: 52}[levels]


def _encoded_msg(scheme, levels, d, n, seed):
    rng = np.random.default_rng(seed)
    cfg = O.Config(scheme, levels, d, 1, 0, 0.0, seed, n)
    g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    return cfg, O.encode(cfg, 0, 0, g)


@pytest.mark.parametrize("scheme,levels", [(O.ORQ, 3), (O.ORQ, 5), (O.ORQ, 9), (O.QSGD, 5),
                                           (O.TERNGRAD, 3), (O.QSGD, 9)])
def test_entropy_is_base_s_stream(scheme, levels):
    """Each bucket's words hold the little-endian bit string sum_i V_i 2^(B i), with
    V_i = sum_k code[g i + k] s^k (built here as one Python integer from the dense codes), and
    the level tables are copied unchanged."""
    g, B = O.entropy_groups(levels)
    for d, n in ((128, 128 * 5 + 3), (512, 512 * 2 + 301)):
        cfg, msg = _encoded_msg(scheme, levels, d, n, 31 + d + levels)
        emsg = O.entropy_pack(cfg, msg)
        _, coff, loff = O.message_layout(cfg)
        _, ecoff, eloff = O.entropy_layout(cfg)
        dw, ew = d * O.bits(levels) // 32, O.entropy_words(cfg)
        words = msg[coff:].view(np.uint32)
        ewords = emsg[ecoff:].view(np.uint32)
        for bk in range(O.num_buckets(cfg)):
            code = O.unpack_bucket(cfg, words[bk * dw:(bk + 1) * dw], d)
            stream = 0
            for i in range(-(-d // g)):
                v = sum(int(code[g * i + k]) * levels ** k for k in range(g) if g * i + k < d)
                stream |= v << (B * i)
            expect = [(stream >> (32 * k)) & 0xffffffff for k in range(ew)]
            assert [int(x) for x in ewords[bk * ew:(bk + 1) * ew]] == expect
        tl = O.num_buckets(cfg) * O.table_len(scheme, levels) * 4
        assert np.array_equal(emsg[eloff:eloff + tl], msg[loff:loff + tl])


@pytest.mark.parametrize("levels", [3, 5, 9])
def test_entropy_roundtrip(levels):
    """unpack(pack(m)) == m for encoded messages, ragged last bucket included; every group
    value is below s^g."""
    g, B = O.entropy_groups(levels)
    for scheme in (O.ORQ, O.QSGD):
        for d, n in ((128, 1), (128, 127), (512, 4096), (1024, 1024 * 2 + 1)):
            cfg, msg = _encoded_msg(scheme, levels, d, n, 7 * d + n)
            emsg = O.entropy_pack(cfg, msg)
            assert np.array_equal(O.entropy_unpack(cfg, emsg), msg)
            ew = O.entropy_words(cfg)
            ewords = emsg.view(np.uint32)
            for bk in range(O.num_buckets(cfg)):
                stream = sum(int(w) << (32 * k) for k, w in enumerate(ewords[bk * ew:(bk + 1) * ew]))
                for i in range(-(-d // g)):
                    assert (stream >> (B * i)) & ((1 << B) - 1) < levels ** g


# ------------------------------------------------------------------------------------------
# Biased baselines ([P3] "Deterministic vs stochastic rounding", "Ternary and binary
# quantization"): QSGD levels with rounding to the nearest level, and the scaled sign
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("levels", [2, 3, 5, 9, 15, 16, 129, 255, 256])
def test_qsgd_nearest_is_nearest_level(levels):
    """Every value goes to a nearest QSGD level (brute force over the levels, up to the
    rounding of the binary32 position); no randomness: seed, step and worker do not matter."""
    rng = np.random.default_rng(70 + levels)
    v = (rng.standard_normal(512) * 1e-3).astype(np.float32)
    outs = []
    for seed, step, worker in ((0, 0, 0), (5, 9, 3)):
        cfg = O.Config(O.QSGD_NEAREST, levels, 512, 1, 0, 0.0, seed, 512)
        code, q, table = O.encode_bucket(cfg, worker, step, 0, v)
        outs.append(code.copy())
        m = float(table[0])
        assert m == float(np.abs(v).max())
        lv = np.array([m * (2 * k - (levels - 1)) / (levels - 1) for k in range(levels)])
        dist = np.abs(lv[None, :] - v.astype(np.float64)[:, None])
        best = dist.min(axis=1)
        got = np.abs(q.astype(np.float64) - v)
        assert np.all(got <= best + 1e-6 * m)
        assert np.array_equal(q, np.array([O.dequant(cfg, table, int(c)) for c in code], dtype=np.float32))
        # the same bracket as stochastic QSGD: the code is k or k + 1
        ks = np.clip(np.trunc((v / np.float32(m) + 1) * (levels - 1) / 2), 0, levels - 2)
        assert np.all((code == ks) | (code == ks + 1))
    assert np.array_equal(outs[0], outs[1])


def test_int8_levels_are_symmetric_integers():
    """[P3] core mechanism: INT8 maps each value to an 8-bit integer with a scale, for a 4x
    compression.  Reading: QSGD with 255 levels, m * (2k - 254) / 254 = m * (k - 127) / 127,
    i.e. the integers -127 .. 127 times m / 127 (zero included), nearest rounding; 8-bit codes."""
    rng = np.random.default_rng(255)
    v = (rng.laplace(0, 1e-3, 512)).astype(np.float32)
    cfg = O.Config(O.QSGD_NEAREST, 255, 512, 1, 0, 0.0, 0, 512)
    assert O.bits(255) == 8
    code, q, table = O.encode_bucket(cfg, 0, 0, 0, v)
    m = float(table[0])
    for c in np.unique(code):
        lvl = O.dequant(cfg, table, int(c))
        assert abs(lvl - m * (int(c) - 127) / 127) <= 2 ** -23 * m
    assert O.dequant(cfg, table, 127) == 0.0
    x = v.astype(np.float64) / m * 127          # nearest integer in -127 .. 127
    near = np.rint(x)
    off = np.abs(x - near) < 0.5 - 1e-3         # away from half-way points
    assert np.array_equal(code[off].astype(int) - 127, near[off].astype(int))
    total, _, _ = O.message_layout(O.Config(O.QSGD_NEAREST, 255, 512, 1, 0, 0.0, 0, 512 * 64))
    assert 32 * 512 * 64 / (8 * total) > 3.9       # about 4x over fp32 with the scale table


def test_qsgd_nearest_ties_go_up():
    """Values exactly half-way between two levels (position y = k + 1/2) take the upper one."""
    v = np.zeros(512, dtype=np.float32)
    v[0] = 1.0                          # m = 1; s = 5: levels -1, -0.5, 0, 0.5, 1, h = 2
    v[1], v[2], v[3], v[4] = 0.25, -0.75, 0.75, -0.25   # y = 2.5, 0.5, 3.5, 1.5
    cfg = O.Config(O.QSGD_NEAREST, 5, 512, 1, 0, 0.0, 0, 512)
    code, q, _ = O.encode_bucket(cfg, 0, 0, 0, v)
    assert list(code[:5]) == [4, 3, 1, 4, 2]
    assert list(q[1:5]) == [0.5, -0.5, 1.0, 0.0]


def test_sign_scale_is_mean_abs():
    """m1 is the binary32 value nearest the exact mean of |u| (checked with rationals), to
    within one ulp (the fixed-point sum carries 45 fraction bits below the largest magnitude)."""
    rng = np.random.default_rng(80)
    for n, scale in ((512, 1e-3), (300, 1e-30), (128, 3e5), (1, 1.0)):
        u = (rng.standard_normal(n) * scale).astype(np.float32)
        exact = sum(Fraction(float(abs(x))) for x in u) / n
        m1 = O.sign_scale(u)
        assert abs(Fraction(float(m1)) - exact) <= Fraction(float(np.spacing(np.float32(m1))))
    assert O.sign_scale(np.zeros(64, np.float32)) == 0.0


def test_signsgd_codes_and_levels():
    """Code 1 for u >= 0 (both zeros included), levels {-m1, +m1}; m1 minimises the squared
    error among scales of the same signs (checked against neighbouring binary32 scales)."""
    rng = np.random.default_rng(81)
    v = (rng.standard_normal(512) * 1e-3).astype(np.float32)
    v[3], v[4] = 0.0, -0.0
    cfg = O.Config(O.SIGNSGD, 2, 512, 1, 0, 0.0, 0, 512)
    code, q, table = O.encode_bucket(cfg, 0, 0, 0, v)
    m1 = O.sign_scale(v)
    assert list(table) == [-m1, m1]
    assert np.array_equal(code, (v >= 0).astype(np.uint8)) and code[3] == 1 and code[4] == 1
    assert np.array_equal(q, np.where(v >= 0, m1, -m1).astype(np.float32))
    sgn = np.where(v >= 0, 1.0, -1.0)
    sse = lambda a: float(np.sum((v.astype(np.float64) - a * sgn) ** 2))
    assert sse(m1) <= sse(np.nextafter(np.float32(m1), np.float32(1))) and \
        sse(m1) <= sse(np.nextafter(np.float32(m1), np.float32(0)))
    # an all-zero bucket quantizes to zeros
    code, q, table = O.encode_bucket(cfg, 0, 0, 0, np.zeros(512, np.float32))
    assert np.all(code == 1) and np.all(q == 0.0) and list(table) == [0.0, 0.0]


def test_signsgd_error_feedback_telescopes():
    """With error feedback the scaled sign loses nothing: sum_t Q_t = sum_t g_t - r_T."""
    rng = np.random.default_rng(82)
    n, d, T = 1000, 128, 8
    cfg = O.Config(O.SIGNSGD, 2, d, 1, 1, 0.0, 0, n)
    r = np.zeros(n, dtype=np.float32)
    gsum = np.zeros(n)
    qsum = np.zeros(n)
    for t in range(T):
        g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
        gsum += g
        msg = O.encode(cfg, 0, t, g, r)
        qsum += O.decode_accumulate(cfg, [msg]).astype(np.float64)
    assert np.allclose(qsum, gsum - r, atol=1e-8)


# ------------------------------------------------------------------------------------------
# QSGD as published (l2 scaling) and Elias integer coding ([P3] "QSGD")
# ------------------------------------------------------------------------------------------
def test_l2_scale_is_norm():
    """m = ||u||_2 from fixed-point sums with 20 fraction bits below max|u|: within 2^-15 of the
    exact norm (checked with rationals), and never below max|u| by more than that."""
    rng = np.random.default_rng(90)
    for n, scale in ((512, 1e-3), (128, 1e-30), (300, 5e4), (1, 2.0)):
        u = (rng.standard_normal(n) * scale).astype(np.float32)
        exact = math.sqrt(float(sum(Fraction(float(x)) ** 2 for x in u)))
        m = O.l2_scale(u)
        assert abs(m - exact) <= 2 ** -15 * exact
        assert m >= float(np.abs(u).max()) * (1 - 2 ** -15)
    assert O.l2_scale(np.zeros(16, np.float32)) == 0.0


def test_qsgd_l2_levels_and_unbiased():
    """QSGD-l2 uses m = ||u||_2 as its scale: table m, levels m (2k - (s-1))/(s-1), and the
    rounding is unbiased (Monte Carlo over 4000 steps)."""
    rng = np.random.default_rng(91)
    v = (rng.standard_normal(128) * 1e-3).astype(np.float32)
    cfg = O.Config(O.QSGD_L2, 3, 128, 1, 0, 0.0, 5, 128)
    _, _, table = O.encode_bucket(cfg, 0, 0, 0, v)
    assert table[0] == O.l2_scale(v)
    acc = np.zeros(128)
    T = 4000
    for t in range(T):
        _, q, _ = O.encode_bucket(cfg, 0, t, 0, v)
        acc += q
    m = float(table[0])
    # each element's variance is at most m^2 / 4 per step
    assert np.all(np.abs(acc / T - v) <= 5 * (m / 2) / math.sqrt(T))


def _gamma_table():
    return {int(r[0]): r[1] for r in _rows("elias_gamma.txt")}


def _elias_stream_bits(codes, s):
    """Concatenated codewords of the codes' symbols, from the golden table (x <= 17)."""
    tab = _gamma_table()
    z0 = (s - 1) // 2
    out = []
    for c in codes:
        z = int(c) - z0
        x = 2 * z + 1 if z >= 0 else -2 * z
        out.append(tab[x])
    return "".join(out)


def test_elias_gamma_lengths_match_table():
    for x, w in _gamma_table().items():
        assert O.elias_gamma_len(x) == len(w)


@pytest.mark.parametrize("scheme,levels", [(O.QSGD, 5), (O.TERNGRAD, 3), (O.QSGD_NEAREST, 9),
                                           (O.QSGD_L2, 3), (O.QSGD_L2, 15), (O.QSGD, 15)])
def test_elias_stream_offsets_and_round_trip(scheme, levels):
    """The stream is the codewords of every valid code in order (built here from the golden
    table), the header holds T and each bucket's first bit, the level tables are copied, and
    unpacking gives the dense message back."""
    for d, n in ((128, 128 * 3 + 5), (512, 512 * 2)):
        rng = np.random.default_rng(d + levels + scheme)
        cfg = O.Config(scheme, levels, d, 1, 0, 0.0, 3, n)
        g = (rng.laplace(0, 1e-3, n)).astype(np.float32)
        msg = O.encode(cfg, 0, 1, g)
        emsg, used = O.elias_pack(cfg, msg)
        cap, ooff, toff, soff = O.elias_layout(cfg)
        nb = O.num_buckets(cfg)
        _, coff, loff = O.message_layout(cfg)
        dw = d * O.bits(levels) // 32
        words = msg[coff:].view(np.uint32)
        bits, offs = "", []
        for bk in range(nb):
            nv = min(d, n - bk * d)
            offs.append(len(bits))
            bits += _elias_stream_bits(O.unpack_bucket(cfg, words[bk * dw:(bk + 1) * dw], nv), levels)
        T = int(emsg[:8].view(np.uint64)[0])
        assert T == len(bits)
        assert list(emsg[ooff:ooff + 8 * nb].view(np.uint64)) == offs
        stream = 0
        for k, ch in enumerate(bits):
            if ch == "1":
                stream |= 1 << k
        nwords = (T + 31) // 32
        got = emsg[soff:soff + 4 * nwords].view(np.uint32)
        assert [int(x) for x in got] == [(stream >> (32 * k)) & 0xffffffff for k in range(nwords)]
        assert not emsg[soff + 4 * nwords:].any()
        assert used == soff + -(-4 * nwords // 16) * 16
        L = O.table_len(scheme, levels)
        assert np.array_equal(emsg[toff:toff + 4 * L * nb], msg[loff:loff + 4 * L * nb])
        assert np.array_equal(O.elias_unpack(cfg, emsg), msg)


def test_elias_unsupported():
    for scheme, levels in ((O.ORQ, 5), (O.QSGD, 4), (O.BINGRAD_B, 2), (O.SIGNSGD, 2), (O.QSGD_L2, 2)):
        assert O.elias_layout(O.Config(scheme, levels, 512, 1, 0, 0.0, 0, 1000)) is None


def test_elias_expected_length_qsgd_l2():
    """QSGD-l2 with 3 levels: element i is non-zero with probability |u_i| / m, so its codeword
    has 1 + 2 |u_i| / m bits on average; the realised stream length over 50 steps agrees within
    five standard deviations."""
    rng = np.random.default_rng(92)
    d, n, steps = 512, 512 * 8, 50
    g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    cfg = O.Config(O.QSGD_L2, 3, d, 1, 0, 0.0, 11, n)
    mean = var = 0.0
    for bk in range(n // d):
        u = g[bk * d:(bk + 1) * d]
        p = np.abs(u.astype(np.float64)) / O.l2_scale(u)
        mean += float(np.sum(1 + 2 * p))
        var += float(np.sum(4 * p * (1 - p)))
    total = 0
    for t in range(steps):
        emsg, _ = O.elias_pack(cfg, O.encode(cfg, 0, t, g))
        total += int(emsg[:8].view(np.uint64)[0])
    assert abs(total - steps * mean) <= 5 * math.sqrt(steps * var)
    assert total / (steps * n) < 1.1   # about 1.06 bits per element against 2 for the dense codes


@pytest.mark.parametrize("scheme,levels", [(O.ORQ, 5), (O.QSGD, 3), (O.BINGRAD_B, 2), (O.SIGNSGD, 2)])
def test_fused_bucket_is_a_slice_of_the_step(scheme, levels):
    """The per-bucket step (used to check sampled buckets of large workloads) gives, for every
    bucket, exactly the slice of the whole-vector step: the average, the new residuals, the
    packed words and the level tables; with error feedback over two steps.  (The whole-vector
    step is built from the per-bucket one; its arithmetic is pinned separately against encode
    followed by decode, which share no code with it.  This checks the per-bucket interface:
    slicing, the ragged last bucket and the residual chain.)"""
    rng = np.random.default_rng(95 + scheme)
    d, n, W = 128, 128 * 3 + 50, 3
    cfg = O.Config(scheme, levels, d, W, 1, 0.0, 8, n)
    rs = [np.zeros(n, np.float32) for _ in range(W)]
    r_b = {b: [np.zeros(min(d, n - b * d), np.float32) for _ in range(W)] for b in range(O.num_buckets(cfg))}
    words = d * O.bits(levels) // 32
    L = O.table_len(scheme, levels)
    _, coff, loff = O.message_layout(cfg)
    for t in range(2):
        gs = [(rng.laplace(0, 1e-3, n)).astype(np.float32) for _ in range(W)]
        avg, msgs = O.fused_step(cfg, t, gs, rs)
        for b in range(O.num_buckets(cfg)):
            lo, hi = b * d, min(n, (b + 1) * d)
            a_b, r_new, w_b, t_b = O.fused_bucket(cfg, t, b, [g[lo:hi] for g in gs], r_b[b])
            assert np.array_equal(a_b.view(np.uint32), avg[lo:hi].view(np.uint32))
            for w in range(W):
                assert np.array_equal(r_new[w].view(np.uint32), rs[w][lo:hi].view(np.uint32))
                assert np.array_equal(w_b[w], msgs[w][coff + 4 * words * b:coff + 4 * words * (b + 1)].view(np.uint32))
                assert np.array_equal(t_b[w].view(np.uint32), msgs[w][loff + 4 * L * b:loff + 4 * L * (b + 1)].view(np.uint32))
            r_b[b] = r_new


# ------------------------------------------------------------------------------------------
# TernGrad with one scale per parameter tensor ([P3] "Ternary and binary quantization")
# ------------------------------------------------------------------------------------------
def test_tg_layer_equals_terngrad_when_every_tensor_is_a_bucket():
    """With the tensors cut exactly at the bucket boundaries (the last one ragged), one scale per
    tensor is one scale per bucket: codes, scales, residuals and average equal TernGrad's."""
    rng = np.random.default_rng(41)
    for d, n in ((128, 5 * 128 + 9), (512, 3 * 512)):
        off = list(range(0, n, d)) + [n]
        cfg = O.Config(O.TERNGRAD, 3, d, 2, 1, 0.0, 7, n)
        gs = [(rng.laplace(0, 1e-3, n)).astype(np.float32) for _ in range(2)]
        ra = [np.zeros(n, np.float32) for _ in range(2)]
        rb = [np.zeros(n, np.float32) for _ in range(2)]
        ma = [O.tg_layer_encode(cfg, off, w, 3, gs[w], ra[w]) for w in range(2)]
        mb = [O.encode(cfg, w, 3, gs[w], rb[w]) for w in range(2)]
        _, _, soff = O.tg_layer_layout(cfg, len(off) - 1)
        _, coff, loff = O.message_layout(cfg)
        for w in range(2):
            assert np.array_equal(ma[w][:soff], mb[w][:loff])  # the codes regions
            nb = len(off) - 1
            assert np.array_equal(ma[w][soff:soff + 4 * nb].view(np.float32), mb[w][loff:loff + 4 * nb].view(np.float32))
            assert np.array_equal(ra[w], rb[w])
        assert np.array_equal(O.tg_layer_decode_accumulate(cfg, off, ma), O.decode_accumulate(cfg, mb))


def _tensor_offsets(rng, n, small=True):
    sizes = []
    while sum(sizes) < n:
        sizes.append(int(rng.choice([64, 37, 1000, 2304, 9, 4096])) if small else 4096)
    off = np.concatenate([[0], np.cumsum(sizes)])
    off[-1] = n
    return off[off <= n] if off[-2] < n else np.concatenate([off[off < n], [n]])


def test_tg_layer_scales_levels_and_residual():
    """Each tensor's scale is its largest |v|; every value is sent as -m, 0 or +m of its own
    tensor, on a side of the value's bracket; the residual keeps v - Q(v)."""
    rng = np.random.default_rng(42)
    n, d = 12000, 512
    off = _tensor_offsets(rng, n)
    cfg = O.Config(O.TERNGRAD, 3, d, 1, 1, 0.0, 9, n)
    g = (rng.laplace(0, 1, n) * 10.0 ** rng.uniform(-4, -2, n)).astype(np.float32)
    for t in range(0, len(off) - 1, 2):  # every other tensor has its largest value last
        g[off[t + 1] - 1] = np.float32((-1) ** t * 3.0 * np.abs(g[off[t]:off[t + 1]]).max())
    r0 = (rng.standard_normal(n) * 1e-5).astype(np.float32)
    r = r0.copy()
    msg = O.tg_layer_encode(cfg, off, 0, 1, g, r)
    nseg = len(off) - 1
    _, _, soff = O.tg_layer_layout(cfg, nseg)
    scales = msg[soff:soff + 4 * nseg].view(np.float32)
    v = g + r0
    q = O.tg_layer_decode_accumulate(cfg, off, [msg])   # one worker: the dequantized values
    assert np.array_equal(r, v - q)
    for t in range(nseg):
        seg = slice(off[t], off[t + 1])
        m = np.float32(np.abs(v[seg]).max())
        assert scales[t] == m
        assert np.all(np.isin(q[seg], np.array([-m, 0.0, m], dtype=np.float32)))
        lo = np.where(v[seg] >= 0, 0.0, -m)
        hi = np.where(v[seg] >= 0, m, 0.0)
        assert np.all((q[seg] == lo) | (q[seg] == hi))


def test_tg_layer_unbiased():
    """Stochastic rounding keeps the expectation: the mean over steps tends to v (3 sigma)."""
    rng = np.random.default_rng(43)
    n, d, steps = 600, 128, 400
    off = [0, 50, 250, 600]
    cfg = O.Config(O.TERNGRAD, 3, d, 1, 0, 0.0, 3, n)
    g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    qs = np.stack([O.tg_layer_decode_accumulate(cfg, off, [O.tg_layer_encode(cfg, off, 0, t, g)]) for t in range(steps)])
    v = g.astype(np.float64)
    m = np.concatenate([np.full(off[t + 1] - off[t], np.abs(v[off[t]:off[t + 1]]).max()) for t in range(3)])
    var = np.abs(v) * (m - np.abs(v))            # (b - v)(v - a) for the bracket [0, m] or [-m, 0]
    sure = var <= 1e-9 * m * m                   # at a level (each tensor's largest): no randomness
    assert np.all(qs[:, sure] == np.float32(v[sure]))
    z = (qs.mean(axis=0)[~sure] - v[~sure]) / np.sqrt(var[~sure] / steps)
    assert np.mean(z ** 2) < 1.3
    assert np.abs(z).max() < 5.5
