"""fp64 references for the block-scaled FP4 GEMM and the Quartet epilogue.

Test infrastructure only (see ``oracle/__init__.py``).

Quartet page, "Stage 2: Dedicated Block-Scaled GEMM Kernel":
D = C + (A x SFA) . (B x SFB) with an FP32 accumulator; both operands are
K-major ("TN": A is M x K, B is N x K, D = A B^T).  The reference is the
exact fp64 product of the dequantised operands times the fp64 product of the
two tensor scales; the acceptance bound per element is
|y - y_ref| <= 2^-10 * sum_k |a_k b_k|.
"""
import numpy as np

from . import hadamard as hd
from . import quant as qn

BOUND_REL = 2.0 ** -10


def tensor_scale_product(A, B):
    return float(A.tensor_scale) * float(B.tensor_scale)


def gemm_ref(A, B):
    """(y_ref, bound) for D = dq(A) dq(B)^T, fp64, full matrices."""
    a = qn.dequant_f64(A, with_tensor_scale=False)
    b = qn.dequant_f64(B, with_tensor_scale=False)
    t = tensor_scale_product(A, B)
    y = (a @ b.T) * t
    bound = BOUND_REL * (np.abs(a) @ np.abs(b).T) * abs(t)
    return y, bound


def gemm_ref_sampled(A, B, ii, jj):
    """The same for the sampled output elements (ii[k], jj[k])."""
    t = tensor_scale_product(A, B)
    rows_a = np.unique(ii)
    rows_b = np.unique(jj)
    a = qn.dequant_f64(_take_rows(A, rows_a), with_tensor_scale=False)
    b = qn.dequant_f64(_take_rows(B, rows_b), with_tensor_scale=False)
    ia = np.searchsorted(rows_a, ii)
    ib = np.searchsorted(rows_b, jj)
    prod = a[ia] * b[ib]
    y = prod.sum(axis=1) * t
    bound = BOUND_REL * np.abs(prod).sum(axis=1) * abs(t)
    return y, bound


def _take_rows(qt, rows):
    return qn.QTensor(qt.codes[rows], qt.scales[rows], qt.tensor_scale, qt.fmt)


def quartet_epilogue_ref(y, bound, keep, had_block=32):
    """Quartet page, "Inverse Hadamard and clipping mask correction":
    dx = 16/9 H_g^-1(dx_q (.) M).  The 16/9 is already inside y (the product
    of the two 4/3 tensor scales).  READING: the page defines M as 1 for a
    clipped element yet says the product zeroes clipped elements, so the
    factor applied is ``keep`` = 1 - M (straight-through estimator).  The
    bound propagates through H: sum_j |h_ij| bound_j."""
    keep = keep.astype(np.float64)
    ym = y * keep
    out = hd.inverse_block_h_f64(ym, had_block)
    bm = bound * keep
    n = bm.shape[-1]
    blk = bm.reshape(bm.shape[:-1] + (n // had_block, had_block)).sum(axis=-1)
    out_bound = np.repeat(blk, had_block, axis=-1) / np.sqrt(float(had_block))
    return out, out_bound
