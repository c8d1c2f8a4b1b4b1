"""Dense orthonormal block transforms: DCT-II and DST-II along the inner
dimension, in blocks of k in {16, 32, 64, 128, 256}.

Test infrastructure only (see ``oracle/__init__.py``).

Bridging-the-Gap page (MR-GPTQ / QuTLASS), "Block-Wise Hadamard Rotation"
and its appendix on linear transforms (Tables 13-14): the forward-pass
rotation of a k-block may be any orthogonal transform -- Hadamard, DCT, DST
or GSR -- at block sizes 16 to 256; the page sweeps them for MXFP4 / NVFP4
RTN and GPTQ.

READINGS (the page names the transforms, not their definitions):
* DCT = the orthonormal DCT-II, C[i, j] = f_i cos(pi (2j + 1) i / (2k)),
  f_0 = sqrt(1/k), f_i = sqrt(2/k); DST = the orthonormal DST-II,
  S[i, j] = g_i sin(pi (2j + 1)(i + 1) / (2k)), g_{k-1} = sqrt(1/k),
  g_i = sqrt(2/k) (the textbook types of the same names; both orthonormal).
* GSR is named but not defined on the pages, so it is not built.
* fp64 matrix entries: cos(pi m / (2k)) is evaluated only for the reduced
  angle index m in [0, k] (every entry is +-1 times one of these, by the
  period 4k and the reflections cos(pi - t) = -cos t, sin t = cos(pi/2 - t));
  the angle is fp64(pi) * m / (2k), rounded twice; the entry is one fp64
  product f_i * (+-cos), rounded once to fp32 for the fp32 transform.
* fp32 evaluation order: y_i = pairwise tree over j of fp32(M[i, j] * x_j)
  (level 0 adds j = (2m, 2m + 1), then adjacent pair sums, ...), every
  multiply and add rounded to fp32 (no fused multiply-add), as the other
  sums of this oracle.
"""
import numpy as np

from . import formats as fm

F32 = np.float32
KINDS = ("dct2", "dst2")


def _cos_table(k):
    """cos(pi m / (2k)) for m = 0..k in fp64, from the fp64 angle
    fp64(pi) * m / (2k)."""
    m = np.arange(k + 1, dtype=np.float64)
    return np.cos(np.pi * m / (2.0 * k))


def _signed_cos(m, k, tab):
    """cos(pi m / (2k)) for any integer m >= 0, through the table: reduce m
    mod 4k, then cos(pi - t) = -cos(t) and cos(2 pi - t) = cos(t)."""
    m = np.asarray(m, dtype=np.int64) % (4 * k)
    m = np.where(m > 2 * k, 4 * k - m, m)              # cos(2 pi - t) = cos t
    neg = m > k
    m = np.where(neg, 2 * k - m, m)                     # cos(pi - t) = -cos t
    v = tab[m]
    return np.where(neg, -v, v)


def dct2_matrix(k):
    """Orthonormal DCT-II matrix (fp64), y = C x."""
    tab = _cos_table(k)
    i = np.arange(k)[:, None]
    j = np.arange(k)[None, :]
    c = _signed_cos((2 * j + 1) * i, k, tab)
    f = np.where(i == 0, np.sqrt(1.0 / k), np.sqrt(2.0 / k))
    return f * c


def dst2_matrix(k):
    """Orthonormal DST-II matrix (fp64), y = S x; the sine is the cosine of
    the complementary angle, sin(pi m / (2k)) = cos(pi (k - m) / (2k))."""
    tab = _cos_table(k)
    i = np.arange(k)[:, None]
    j = np.arange(k)[None, :]
    m = (2 * j + 1) * (i + 1)
    c = _signed_cos(k - m + 8 * k * k, k, tab)         # + a multiple of 4k keeps the index non-negative
    g = np.where(i == k - 1, np.sqrt(1.0 / k), np.sqrt(2.0 / k))
    return g * c


def matrix_f64(kind, k):
    if kind == "dct2":
        return dct2_matrix(k)
    if kind == "dst2":
        return dst2_matrix(k)
    raise ValueError(kind)


def matrix_f32(kind, k):
    """The fp32 entries the transform multiplies by (each rounded once)."""
    return matrix_f64(kind, k).astype(F32)


def block_transform_f32(x, kind, k, rows_per_chunk=64):
    """y = M x per k-block of the last axis of fp32 ``x`` (2-D, rows x cols,
    cols a multiple of k): y_i = pairwise tree over j of fp32(M[i, j] x_j)."""
    x = np.asarray(x, dtype=F32)
    rows, cols = x.shape
    assert cols % k == 0
    m = matrix_f32(kind, k)
    out = np.empty((rows, cols), dtype=F32)
    for r0 in range(0, rows, rows_per_chunk):
        xb = x[r0:r0 + rows_per_chunk].reshape(-1, cols // k, 1, k)      # (r, blocks, 1, j)
        prod = (m[None, None, :, :] * xb).astype(F32)                     # (r, blocks, i, j)
        out[r0:r0 + rows_per_chunk] = fm.pairwise_sum(prod).reshape(-1, cols)
    return out


def block_transform_f64(x, kind, k):
    """The exact-in-fp64 reference y = M x (M in fp64) per k-block."""
    x = np.asarray(x, dtype=np.float64)
    rows, cols = x.shape
    xb = x.reshape(rows, cols // k, k)
    return (xb @ matrix_f64(kind, k).T).reshape(rows, cols)
