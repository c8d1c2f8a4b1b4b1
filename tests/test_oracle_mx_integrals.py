"""Pins of the oracle's MXFP4 RTN and stochastic-rounding errors, and of its
NVFP4 RTN error, to their expected values on Gaussian data, computed by
numerical integration from the formats' definitions alone (no oracle code).
MXFP4: groups of 32 iid N(0, 1)
values (the same after an orthonormal 32-point Hadamard, which maps iid
N(0, 1) to iid N(0, 1)), the shared scale 2^(floor(log2 M) - 2) of the
group maximum M (the OCP rule of the Quartet and Bridging-the-Gap pages),
and the E2M1 grid {0, 0.5, 1, 1.5, 2, 3, 4, 6}.

Given M = m, one element has |x| = m and the other 31 are iid |N(0, 1)|
truncated to [0, m]; M has density 32 (2 Phi(m) - 1)^31 2 phi(m).  Per
element:
* RTN: the squared distance to the nearest grid point times s (values
  above 6 s saturate to 6 s);
* SR with the Quartet backward's 3/4 pre-scale (v = 3 x / (4 s) <= 6, so
  no clipping) and the 4/3 carried back: unbiased, with conditional
  variance (4 s / 3)^2 (v - lo)(hi - v) between the neighbouring grid
  points lo <= v <= hi.
NVFP4 RTN: groups of 16, the tensor scale s_T = amax / (6 x 256) of the
sample, the group scale d = s_T x E4M3(M / (6 s_T)) (round to nearest,
3 mantissa bits), elements rounded to the grid times d (saturating at 6 d,
which the max element can exceed when E4M3 rounds its scale down).  NVFP4
SR: the 16/17 guard in both scales, unbiased SR of y / d (variance
d^2 (v - lo)(hi - v)), no clipping.
The oracle's Monte Carlo means over 2^20 elements must match within their
sampling error (1%)."""
import math

import numpy as np
from scipy import integrate

from oracle import hadamard as hd
from oracle import quant as qn

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
MIDS = (GRID[1:] + GRID[:-1]) / 2


def _phi(y):
    return math.exp(-0.5 * y * y) / math.sqrt(2 * math.pi)


def _cdf2(m):
    """P(|x| <= m) = 2 Phi(m) - 1."""
    return math.erf(m / math.sqrt(2.0))


def _rtn_err(y, s):
    """Squared RTN error of y >= 0 at scale s (saturating at 6 s)."""
    v = y / s
    if v >= 6.0:
        return (y - 6.0 * s) ** 2
    g = GRID[np.searchsorted(MIDS, v)]
    return (y - g * s) ** 2


def _sr_err(y, s):
    """Expected squared error of unbiased SR of v = 3 y / (4 s) on the grid,
    carried back by 4 s / 3."""
    v = 0.75 * y / s
    i = min(int(np.searchsorted(GRID, v, side="right")) - 1, len(GRID) - 2)
    lo, hi = GRID[i], GRID[i + 1]
    return (4.0 * s / 3.0) ** 2 * (v - lo) * (hi - v)


def _breaks(s, m, kind):
    """Points in [0, m] where the error function changes its formula."""
    pts = (MIDS * s) if kind == "rtn" else (GRID[1:-1] * 4.0 * s / 3.0)
    extra = [6.0 * s] if kind == "rtn" else []
    return [0.0] + [p for p in list(pts) + extra if 0.0 < p < m] + [m]


def _expected_mse(kind):
    err = _rtn_err if kind == "rtn" else _sr_err

    def per_group(m):
        s = 2.0 ** (math.floor(math.log2(m)) - 2)
        pts = _breaks(s, m, kind)
        inner = sum(integrate.quad(lambda y: err(y, s) * 2.0 * _phi(y), a, b, epsabs=1e-13)[0]
                    for a, b in zip(pts[:-1], pts[1:]))
        return (err(m, s) + 31.0 * inner / _cdf2(m)) / 32.0

    def dens(m):
        return 32.0 * _cdf2(m) ** 31 * 2.0 * _phi(m)

    total = 0.0
    for k in range(-6, 3):                                # m in [2^k, 2^(k+1)): the scale is fixed
        a, b = 2.0 ** k, min(2.0 ** (k + 1), 8.0)
        total += integrate.quad(lambda m: dens(m) * per_group(m), a, b, epsabs=1e-12, limit=200)[0]
    return total                                         # P(M < 2^-6) and P(M > 8) are below 1e-30


def _gauss(seed):
    return np.random.default_rng(seed).standard_normal((1024, 1024)).astype(np.float32)


def _mse(qt, x):
    return float(np.mean((qn.dequant_f64(qt) - x.astype(np.float64)) ** 2))


def test_mxfp4_rtn_mean_squared_error_is_the_integral():
    want = _expected_mse("rtn")
    x = _gauss(11)
    got = _mse(qn.mxfp4_rtn(x), x)
    assert abs(got - want) <= 0.01 * want
    xr = hd.block_transform(x, 32, False)                # still iid N(0, 1)
    assert abs(_mse(qn.mxfp4_rtn(xr), xr) - want) <= 0.01 * want


def test_mxfp4_sr_mean_squared_error_is_the_integral():
    want = _expected_mse("sr")
    x = _gauss(12)
    got = _mse(qn.mxfp4_sr(x, 5, 1), x)
    assert abs(got - want) <= 0.01 * want
    assert want > _expected_mse("rtn")                   # the ordering the Quartet page states


def _nv_sr_err(y, d):
    """Expected squared error of unbiased SR of y / d on the grid (no clipping), times d^2."""
    v = y / d
    i = min(int(np.searchsorted(GRID, v, side="right")) - 1, len(GRID) - 2)
    lo, hi = GRID[i], GRID[i + 1]
    return d * d * (v - lo) * (hi - v)


def _nvfp4_expected_mse(s_t, group_div, kind):
    """Groups of 16: the group scale d = s_T x E4M3(M / (group_div s_T)); RTN
    (saturating at 6 d) or SR (the 16/17 guard keeps y / d within 6)."""
    err = _rtn_err if kind == "rtn" else _nv_sr_err

    def dens(m):
        return 16.0 * _cdf2(m) ** 15 * 2.0 * _phi(m)

    def piece(a, b, d):
        def per_group(m):
            marks = list(MIDS * d) + [6.0 * d] if kind == "rtn" else list(GRID[1:-1] * d)
            pts = [0.0] + [p for p in marks if 0.0 < p < m] + [m]
            inner = sum(integrate.quad(lambda y: err(y, d) * 2.0 * _phi(y), lo, hi, epsabs=1e-14)[0]
                        for lo, hi in zip(pts[:-1], pts[1:]))
            return (err(m, d) + 15.0 * inner / _cdf2(m)) / 16.0
        return integrate.quad(lambda m: dens(m) * per_group(m), a, b, epsabs=1e-13, limit=100)[0]

    # every normal E4M3 value and the interval of t = M / (group_div s_T) that rounds to it
    vals = sorted({2.0 ** e * (1.0 + mm / 8.0) for e in range(-6, 9) for mm in range(8)
                   if 2.0 ** e * (1.0 + mm / 8.0) <= 448.0})
    total = 0.0
    for i, v in enumerate(vals):
        t_lo = 0.5 * (vals[i - 1] + v) if i else v
        t_hi = 0.5 * (v + vals[i + 1]) if i + 1 < len(vals) else 2.0 * v
        a, b = group_div * s_t * t_lo, min(group_div * s_t * t_hi, 9.0)
        if a >= b or b < 0.05:                           # P(M < 0.05) < 1e-20 for 16 values
            continue
        total += piece(a, b, v * s_t)
    return total


def test_nvfp4_rtn_mean_squared_error_is_the_integral():
    x = _gauss(13)
    amax = np.float32(np.max(np.abs(x)))
    s_t = float(np.float32(amax / np.float32(6.0 * 256.0)))
    want = _nvfp4_expected_mse(s_t, 6.0, "rtn")
    got = _mse(qn.nvfp4_rtn(x), x)
    assert abs(got - want) <= 0.01 * want


def test_nvfp4_sr_mean_squared_error_is_the_integral():
    """The Quartet II page's standard NVFP4 SR: s_T = amax / (6 x 16/17 x 448),
    group scale E4M3(M / (6 x 16/17 x s_T))."""
    x = _gauss(14)
    amax = np.float32(np.max(np.abs(x)))
    g = 6.0 * 16.0 / 17.0
    s_t = float(np.float32(amax / np.float32(g * 448.0)))
    want = _nvfp4_expected_mse(s_t, float(np.float32(g)), "sr")
    got = _mse(qn.nvfp4_sr(x, 3, 1), x)
    assert abs(got - want) <= 0.01 * want
