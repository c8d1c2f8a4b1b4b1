"""Pins of the oracle's forward-only variants of the Bridging-the-Gap page:
the DCT-II / DST-II block transforms (appendix on linear transforms, Tables
13-14) and the MXFP4 scale fit (MXFP4-dagger, "MXFP Scale Fitting",
Appendix H).  The transforms are pinned to scipy's orthonormal DCT / DST and
to orthonormality; the fp32 evaluation to its exact fp64 value within the
error bound of a pairwise sum, and to an element-by-element loop on a small
case.  The scale fit is pinned to its definition: nearest level in the log
domain (brute force), the extreme groups at levels 0 and 255, the closed
form of a tensor whose group scales are all equal, the scale within half a
level of the AbsMax scale, and a smaller error than the power-of-two rule."""
import numpy as np
import pytest
import scipy.fft as sf

from fp4_microscaled_quantized_b200 import synthetic as syn
from oracle import formats as fm
from oracle import quant as qn
from oracle import transforms as tr

F32 = np.float32
BLOCKS = (16, 32, 64, 128, 256)


@pytest.mark.parametrize("k", BLOCKS)
def test_matrices_are_scipys_orthonormal_dct_and_dst(k):
    eye = np.eye(k)
    np.testing.assert_allclose(tr.dct2_matrix(k), sf.dct(eye, type=2, norm="ortho", axis=0), rtol=0, atol=1e-15)
    np.testing.assert_allclose(tr.dst2_matrix(k), sf.dst(eye, type=2, norm="ortho", axis=0), rtol=0, atol=1e-15)
    for kind in tr.KINDS:
        m = tr.matrix_f64(kind, k)
        np.testing.assert_allclose(m @ m.T, eye, rtol=0, atol=1e-14)


def test_matrix_closed_forms():
    """Entries written out: DCT-II row 0 is 1/sqrt(k); DST-II row k-1 is
    (-1)^j / sqrt(k); DCT-II [1, 0] = sqrt(2/k) cos(pi / (2k))."""
    k = 16
    c, s = tr.dct2_matrix(k), tr.dst2_matrix(k)
    np.testing.assert_allclose(c[0], np.full(k, 0.25), rtol=0, atol=1e-16)
    np.testing.assert_allclose(s[k - 1], 0.25 * (-1.0) ** np.arange(k), rtol=0, atol=1e-16)
    assert c[1, 0] == pytest.approx(np.sqrt(2.0 / k) * np.cos(np.pi / 32), abs=1e-16)


@pytest.mark.parametrize("kind", tr.KINDS)
@pytest.mark.parametrize("k", BLOCKS)
def test_basis_vectors_give_the_fp32_columns(kind, k):
    """The transform of e_j is column j of the fp32 matrix exactly (one
    non-zero product, the rest of the tree adds zeros)."""
    x = np.zeros((k, 2 * k), dtype=F32)
    for j in range(k):
        x[j, k + j] = 1.0
    y = tr.block_transform_f32(x, kind, k)
    m32 = tr.matrix_f32(kind, k)
    np.testing.assert_array_equal(y[:, :k], 0.0)
    np.testing.assert_array_equal(y[:, k:].T, m32)


@pytest.mark.parametrize("kind", tr.KINDS)
@pytest.mark.parametrize("k", BLOCKS)
def test_fp32_transform_within_its_error_bound(kind, k):
    """|y32 - M x| <= (2^-24 (1 + log2 k) + rounding of M) sum|M_ij x_j|
    against the exact fp64 product with the fp64 matrix."""
    x = syn.bf16_bits_to_f32(syn.gaussian((8, 2 * k), 1.0, seed=k))
    y = tr.block_transform_f32(x, kind, k).astype(np.float64)
    ref = tr.block_transform_f64(x, kind, k)
    m = np.abs(tr.matrix_f64(kind, k))
    mag = (np.abs(x.astype(np.float64)).reshape(8, 2, k) @ m.T).reshape(8, 2 * k)
    bound = (2.0 ** -24) * (2 + np.log2(k)) * mag
    assert np.all(np.abs(y - ref) <= bound)


def test_evaluation_order_is_the_pairwise_tree():
    """k = 16 written as an explicit loop: products, then levels of adjacent sums."""
    x = syn.bf16_bits_to_f32(syn.gaussian((3, 32), 1.0, seed=9))
    m = tr.matrix_f32("dct2", 16)
    want = np.empty_like(x)
    for r in range(3):
        for b in range(2):
            for i in range(16):
                level = [F32(m[i, j] * x[r, 16 * b + j]) for j in range(16)]
                while len(level) > 1:
                    level = [F32(level[2 * t] + level[2 * t + 1]) for t in range(len(level) // 2)]
                want[r, 16 * b + i] = level[0]
    np.testing.assert_array_equal(fm.f32_bits(tr.block_transform_f32(x, "dct2", 16)), fm.f32_bits(want))


# ------------------------------------------------------------ scale fit --
def _gauss_mixed(rows, cols, seed):
    """N(0, 1) rows with a per-row scale spread over 2^-8 .. 2^8, so group
    scales cover many binades."""
    g = syn.bf16_bits_to_f32(syn.gaussian((rows, cols), 1.0, seed=seed))
    sc = np.exp2(np.linspace(-8, 8, rows)).astype(F32)[:, None]
    return (g * sc).astype(F32)


def test_fit_levels_are_the_nearest_in_log_domain():
    x = _gauss_mixed(48, 256, 3)
    f = qn.mxfp4_fit(x)
    s = (np.abs(x).reshape(48, -1, 32).max(-1) / F32(6.0)).astype(F32).astype(np.float64)
    v = (np.log2(s) - f.l_min) / f.alpha
    brute = np.clip(np.floor(v + 0.5), 0, 255).astype(np.int64)
    # equal except where the fp32 boundary rounding sits within 1e-6 levels of a tie
    diff = f.q.astype(np.int64) != brute
    assert np.all(np.abs(v[diff] - np.round(v[diff] - 0.5) - 0.5) < 1e-6)
    assert diff.mean() < 1e-3


def test_fit_extreme_groups_and_table_ends():
    x = _gauss_mixed(48, 256, 4)
    f = qn.mxfp4_fit(x)
    s = (np.abs(x).reshape(48, -1, 32).max(-1) / F32(6.0)).astype(F32)
    assert f.q[s == s.min()].max() == 0 and f.q[s == s.max()].min() == 255
    assert f.table[0] == s.min() and f.table[255] == s.max()       # 2^(log2 s) rounds back to s
    assert np.all(np.diff(f.table.astype(np.float64)) > 0) and np.all(np.diff(f.thresholds.astype(np.float64)) > 0)
    # every group's scale lies within half a level (2^(alpha / 2)) of its AbsMax scale
    d = f.table[f.q.astype(np.int64)].astype(np.float64)
    r = np.abs(np.log2(d / s.astype(np.float64)))
    assert np.all(r <= f.alpha / 2 + 1e-6)


def test_fit_with_one_scale_is_the_absmax_rule():
    """Every group has the same AbsMax scale s: alpha = 0, every level's
    scale is s (each group counts all 255 boundaries, which equal s, so its
    level is 255; any level would give the same scale), and the codes are
    RTN_E2M1(x * fp32(1/s))."""
    rng = np.random.default_rng(5)
    x = rng.uniform(-5.0, 5.0, (8, 128)).astype(F32)
    x.reshape(8, 4, 32)[:, :, 0] = F32(7.5)               # group max 7.5, s = 1.25
    f = qn.mxfp4_fit(x)
    assert f.alpha == 0.0 and np.all(f.table == F32(1.25)) and np.all(f.q == 255)
    inv = F32(1.0) / F32(1.25)
    np.testing.assert_array_equal(f.codes, fm.rtn_e2m1((x * inv).astype(F32)))


def test_fit_zero_groups_and_empty_tensor():
    x = _gauss_mixed(4, 128, 6)
    x[1, 32:64] = 0.0
    f = qn.mxfp4_fit(x)
    assert f.q[1, 1] == 0 and np.all(f.codes[1, 32:64] == 0)
    z = qn.mxfp4_fit(np.zeros((2, 64), dtype=F32))
    assert np.all(z.codes == 0) and np.all(z.q == 0) and np.all(z.table == F32(1.0))


def test_fit_error_below_the_power_of_two_rule():
    """The page's claim (Appendix H, Table 11): fitted fractional-exponent
    scales quantise with less error than the E8M0 power-of-two rule."""
    x = _gauss_mixed(256, 512, 7)
    fit = np.mean((qn.mxfp4_fit_dequant(qn.mxfp4_fit(x)).astype(np.float64) - x) ** 2 / np.mean(x * x, axis=1,
                                                                                              keepdims=True))
    rtn = np.mean((qn.dequant_f32(qn.mxfp4_rtn(x)).astype(np.float64) - x) ** 2 / np.mean(x * x, axis=1,
                                                                                         keepdims=True))
    assert fit < 0.8 * rtn
