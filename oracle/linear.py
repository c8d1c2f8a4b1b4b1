"""The fully-FP4 linear layer, forward and backward, for the three recipes.

Test infrastructure only (see ``oracle/__init__.py``).

* QUARTET -- Quartet page, "The Complete Quartet Algorithm" (Algorithm 1):
  forward X_h = H32(X), W_h = H32(W), QuEST on MXFP4 (with clip masks),
  Y = GEMM(X_q, W_q); backward G = SR(3/4 RHT32(dY)) against
  SR(3/4 RHT32(W_q^T)) for dX and SR(3/4 RHT32(dY^T)) against
  SR(3/4 RHT32(X_q^T)) for dW, each followed by 16/9 H32^-1( . (.) mask).
* QUARTET2 -- Quartet II page, "The Complete Quartet II Computation Graph":
  forward RTN + Four-Over-Six on NVFP4 (no rotation); backward de-quantise,
  transpose, RHT128 on the inner dimension and MS-EDEN for (E, W^T) and
  (E^T, X^T); no inverse transform.
* RTN -- a single NVFP4 RTN linear layer without rotation.
* NVIDIA -- the NVIDIA recipe the Quartet II page describes ("The
  square-block trade-off"; "Comparison to TetraJet-v2 and the NVIDIA
  recipe"): forward X with native 1x16 RTN scales, W with 16x16 square-block
  RTN scales, no rotation; backward SR; the dX GEMM re-uses the forward Q(W),
  transposed, with dY quantised along N without a rotation (the rotation must
  act on both operands of a GEMM, and W is re-used as it is); the dW GEMM
  rotates both operands (SR of RHT(dY^T) and of RHT(Q(X)^T)).  READINGS: the
  page does not give the dW GEMM's operands beyond "RHT only on the backward
  pass"; X^T is re-quantised from the saved Q(X) as in the other recipes, and
  the rotation block is 16, the square block size.
* TETRAJET2 -- the simplified TetraJet-v2 of the Quartet II page ("Comparison
  to TetraJet-v2 and the NVIDIA recipe"): NVFP4 RTN with native 1x16 scales
  on the forward pass, SR with the RHT on the inner dimension for both
  backward GEMMs, weights and activations re-quantised -- the QUARTET2 graph
  with SR in place of MS-EDEN (READING: the same 128-element rotation, since
  the page names MS-EDEN as the one difference).

READING (seed scheme, the pages name none): every random draw of one
backward step uses key = step_seed; the two GEMMs' rotations use sign tags
GEMM_DX / GEMM_DW (so both operands of a GEMM share the signs, as the
Quartet II page requires); the four SR streams use tensor tags
TAG_E_ROW, TAG_W_T, TAG_E_T, TAG_X_T.
"""
from dataclasses import dataclass

import numpy as np

from . import gemm as gm
from . import quant as qn

GEMM_DX, GEMM_DW = 0, 1
TAG_E_ROW, TAG_W_T, TAG_E_T, TAG_X_T, TAG_X, TAG_W = 1, 2, 3, 4, 5, 6


@dataclass(frozen=True)
class Recipe:
    fmt: int
    fwd_rnd: int
    fwd_had: int
    bwd_rnd: int
    bwd_had: int
    bwd_randomized: bool
    mask_epilogue: bool
    w_rnd: int = -1          # forward rounding of W (-1: fwd_rnd)
    w_reuse: bool = False    # dX GEMM re-uses Q(W)^T; dY quantised without rotation


QUARTET = Recipe(qn.MXFP4, qn.QUEST, 32, qn.SR, 32, True, True)
QUARTET2 = Recipe(qn.NVFP4, qn.FOUR_OVER_SIX, 0, qn.MS_EDEN, 128, True, False)
RTN = Recipe(qn.NVFP4, qn.RTN, 0, qn.RTN, 0, False, False)
TETRAJET2 = Recipe(qn.NVFP4, qn.RTN, 0, qn.SR, 128, True, False)
NVIDIA = Recipe(qn.NVFP4, qn.RTN, 0, qn.SR, 16, True, False, w_rnd=qn.RTN_SQUARE16, w_reuse=True)


def linear_fwd(X, W, r, seed=0):
    """Returns (Y_ref, bound, ctx) with ctx = {"Xq", "Wq"}."""
    Xq = qn.quantize(X, r.fmt, r.fwd_rnd, r.fwd_had, False, seed, 0, TAG_X)
    w_rnd = r.fwd_rnd if r.w_rnd < 0 else r.w_rnd
    Wq = qn.quantize(W, r.fmt, w_rnd, r.fwd_had, False, seed, 0, TAG_W)
    y, b = gm.gemm_ref(Xq, Wq)
    return y, b, {"Xq": Xq, "Wq": Wq}


def bwd_operands(dY, ctx, r, step_seed):
    """The four backward operands, quantised along each GEMM's inner dim."""
    h, rz, s = r.bwd_had, r.bwd_randomized, step_seed
    if r.w_reuse:
        E_row = qn.quantize(dY, r.fmt, r.bwd_rnd, 0, False, s, GEMM_DX, TAG_E_ROW)
        W_t = qn.transpose_square16(ctx["Wq"])
    else:
        E_row = qn.quantize(dY, r.fmt, r.bwd_rnd, h, rz, s, GEMM_DX, TAG_E_ROW)
        W_t = qn.requantize(ctx["Wq"], r.bwd_rnd, h, rz, s, GEMM_DX, TAG_W_T, transpose=True)
    E_t = qn.quantize(dY, r.fmt, r.bwd_rnd, h, rz, s, GEMM_DW, TAG_E_T, transpose=True)
    X_t = qn.requantize(ctx["Xq"], r.bwd_rnd, h, rz, s, GEMM_DW, TAG_X_T, transpose=True)
    return {"E_row": E_row, "W_t": W_t, "E_t": E_t, "X_t": X_t}


def linear_bwd(dY, ctx, r, step_seed):
    """Returns ((dX_ref, dX_bound), (dW_ref, dW_bound), operands)."""
    ops = bwd_operands(dY, ctx, r, step_seed)
    dx, bx = gm.gemm_ref(ops["E_row"], ops["W_t"])
    dw, bw = gm.gemm_ref(ops["E_t"], ops["X_t"])
    if r.mask_epilogue:
        dx, bx = gm.quartet_epilogue_ref(dx, bx, ~ctx["Xq"].mask, r.fwd_had)
        dw, bw = gm.quartet_epilogue_ref(dw, bw, ~ctx["Wq"].mask, r.fwd_had)
    return (dx, bx), (dw, bw), ops


def flops_fwd_bwd(M, N, K):
    return 6.0 * M * N * K
