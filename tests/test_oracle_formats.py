"""Pins of the oracle's number formats against the pages and library routines."""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import formats as fm

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "e2m1_grid.json")))


def test_e2m1_grid_matches_pages():
    vals = fm.decode_e2m1(np.arange(16, dtype=np.uint8))
    assert list(vals[:8]) == GOLD["positive_values"]
    assert list(-vals[8:]) == GOLD["positive_values"]
    assert fm.E2M1_MAX == GOLD["max"]


def test_rtn_e2m1_is_nearest_grid_point_brute_force():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.uniform(-8, 8, 4000), rng.standard_normal(2000) * 0.3]).astype(np.float32)
    codes = fm.rtn_e2m1(v)
    grid = GOLD["positive_values"]
    for x, c in zip(v.tolist(), codes.tolist()):
        a = abs(x)
        dists = [abs(a - g) for g in grid]
        best = min(dists)
        cands = [i for i, d in enumerate(dists) if d == best]
        idx = [i for i in cands if i % 2 == 0][0] if len(cands) > 1 else cands[0]
        want = idx | (8 if (x < 0 and idx != 0) else 0)
        assert c == want, (x, c, want)


def test_rtn_e2m1_ties_dead_zone_saturation():
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    assert fm.decode_e2m1(fm.rtn_e2m1(ties)).tolist() == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]
    dz = np.array([0.2499999, -0.2499999, 1e-30, -0.0], dtype=np.float32)
    assert fm.rtn_e2m1(dz).tolist() == [0, 0, 0, 0]           # dead zone, -0 -> +0
    sat = np.array([6.0, 6.5, 100.0, -7.0, 3e38], dtype=np.float32)
    assert fm.decode_e2m1(fm.rtn_e2m1(sat)).tolist() == [6.0, 6.0, 6.0, -6.0, 6.0]
    with pytest.raises(ValueError):
        fm.rtn_e2m1(np.array([np.nan], dtype=np.float32))


def test_e4m3_table_against_torch():
    codes = np.arange(127, dtype=np.uint8)
    want = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(fm.E4M3_VALUES, want)
    assert fm.E4M3_VALUES[-1] == GOLD["e4m3_max"]


def test_rtn_e4m3_against_torch_conversion():
    rng = np.random.default_rng(1)
    t = np.concatenate([rng.uniform(0, 448, 20000), np.exp(rng.uniform(-12, 6, 20000)),
                        fm.E4M3_VALUES, (fm.E4M3_VALUES[1:] + fm.E4M3_VALUES[:-1]) / 2]).astype(np.float32)
    t = t[t <= 448]
    ours = fm.rtn_e4m3(t)
    ref = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, ref)
    assert fm.rtn_e4m3(np.array([500.0, 1e30], dtype=np.float32)).tolist() == [126, 126]


def _exact_mean_over_u(fn, v, n=1 << 12):
    u = (np.arange(n) + 0.5) / n
    return np.array([np.mean(fm.decode_e2m1(fn(np.full(n, x, np.float32), u)).astype(np.float64))
                     for x in v])


def test_sr_e2m1_exact_expectation():
    v = np.array([0.1, 0.3, 0.75, 1.2, 1.9, 2.2, 3.7, 4.1, 5.99, -2.6, -0.01], dtype=np.float32)
    m = _exact_mean_over_u(fm.sr_e2m1, v)
    np.testing.assert_allclose(m, v.astype(np.float64), atol=2.0 / (1 << 12))
    # values on the grid never move; |v| >= 6 saturates
    g = fm.decode_e2m1(np.arange(16, dtype=np.uint8))
    assert np.array_equal(fm.decode_e2m1(fm.sr_e2m1(g, np.full(16, 0.999))), g)
    assert fm.decode_e2m1(fm.sr_e2m1(np.array([7.0], np.float32), np.array([0.0]))).tolist() == [6.0]


def test_sr_e4m3_expectation_and_subnormal_rtn():
    t = np.array([0.02, 0.3, 1.06, 7.3, 100.1, 300.0], dtype=np.float32)
    n = 1 << 12
    u = (np.arange(n) + 0.5) / n
    for x in t:
        vals = fm.e4m3_value(fm.sr_e4m3(np.full(n, x, np.float32), u))
        assert abs(vals.mean() - float(x)) <= 2.0 / n * float(x)
    small = np.array([2.0 ** -7 * 1.3, 2.0 ** -9 * 0.7], dtype=np.float32)   # E4M3 subnormal range
    assert np.array_equal(fm.sr_e4m3(small, np.array([0.0, 0.0])), fm.rtn_e4m3(small))
    assert fm.sr_e4m3(np.array([448.0, 460.0], np.float32), np.array([0.0, 0.0])).tolist() == [126, 126]


def test_e8m3_round_definition_and_bf16():
    rng = np.random.default_rng(2)
    t = np.exp(rng.uniform(-40, 40, 5000)).astype(np.float32)
    q = fm.e8m3_round(t).astype(np.float64)
    for x, y in zip(t.astype(np.float64)[:500], q[:500]):
        e = math.floor(math.log2(x))
        # candidates with 3 fractional mantissa bits around x
        step = 2.0 ** (e - 3)
        lo = math.floor(x / step) * step
        hi = lo + step
        want = lo if (x - lo < hi - x) or (x - lo == hi - x and (lo / step) % 2 == 0) else hi
        assert y == want
    # exactly representable in bf16: the low 16 fp32 bits are zero
    assert np.all((q.astype(np.float32).view(np.uint32) & 0xFFFF) == 0)
    assert abs(np.max(np.abs(q / t.astype(np.float64) - 1))) <= 1 / 16


def test_pairwise_sum_tree_order():
    a = np.array([1e8, 1.0, -1e8, 1.0, 3.0, 5.0, 7.0, 9.0], dtype=np.float32)
    f = np.float32
    want = f(f(f(a[0] + a[1]) + f(a[2] + a[3])) + f(f(a[4] + a[5]) + f(a[6] + a[7])))
    assert fm.pairwise_sum(a) == want
    rng = np.random.default_rng(3)
    x = rng.standard_normal((100, 128)).astype(np.float32)
    ref = np.array([math.fsum(r) for r in x.astype(np.float64)])
    assert np.max(np.abs(fm.pairwise_sum(x) - ref)) < 1e-5


def test_packing_roundtrip_and_nibble_order():
    codes = np.array([[1, 2, 3, 4, 15, 0, 7, 8]], dtype=np.uint8)
    p = fm.pack_codes(codes)
    assert p.tolist() == [[0x21, 0x43, 0x0F, 0x87]]
    assert np.array_equal(fm.unpack_codes(p), codes)
    m = np.zeros((1, 16), dtype=bool)
    m[0, [0, 3, 9]] = True
    pm = fm.pack_mask(m)
    assert pm.tolist() == [[0b1001, 0b10]]
    assert np.array_equal(fm.unpack_mask(pm, 16), m)
