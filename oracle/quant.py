"""Micro-scaled FP4 quantizers: MXFP4 / NVFP4 x {RTN, QuEST, Four-Over-Six,
SR, MS-EDEN}, NVFP4 square-block RTN and the MSE-optimal scale search, plus
dequantisation and the tensor-core scale layout.

Test infrastructure only (see ``oracle/__init__.py``).

Every function takes the (already transformed) fp32 tensor to quantise,
shaped (rows, cols) with the groups running along ``cols`` (the GEMM's inner
dimension), and follows the pages' steps in their order.  Readings where the
pages are silent are marked READING.
"""
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

from . import formats as fm
from . import hadamard as hd
from . import philox

F32 = np.float32

MXFP4, NVFP4 = 0, 1
RTN, QUEST, FOUR_OVER_SIX, SR, MS_EDEN, RTN_SQUARE16 = 0, 1, 2, 3, 4, 5
GROUP = {MXFP4: 32, NVFP4: 16}

# NVFP4 tensor-scale divisors.
# Quartet II page, "MS-EDEN" Step 2: x_fp32 = amax / (s * 256); the same
# divisor with s = 6 (the E2M1 maximum) is the READING used for the
# deterministic NVFP4 rules (RTN, Four-Over-Six, QuEST), the page's only RTN
# formula; 256 leaves headroom below the E4M3 maximum 448.
NV_RTN_DIV = F32(6.0 * 256.0)
# READING: MS-EDEN clip factor s = 6 (the page never prints s; 6 reproduces
# Table 1's 9.8e-3, the non-clipping 6*16/17 gives about 11e-3).
MS_EDEN_S = F32(6.0)
MS_EDEN_DIV = F32(6.0 * 256.0)
# Quartet II page, "NVFP4 Format and Standard Stochastic Rounding", Step 1/2.
NV_SR_DIV = F32(6.0 * 16.0 / 17.0 * 448.0)
NV_SR_GROUP_DIV = F32(6.0 * 16.0 / 17.0)
# Quartet page, "Backward-Pass Quantization": SR(3/4 G_h), 16/9 after GEMM.
QUARTET_PRESCALE = F32(0.75)
QUARTET_TENSOR_SCALE = F32(4.0 / 3.0)


@dataclass
class QTensor:
    codes: np.ndarray                 # (rows, cols) uint8, unpacked E2M1 codes
    scales: np.ndarray                # (rows, cols // g) uint8 (E8M0 or E4M3)
    tensor_scale: np.float32          # NVFP4 fp32 scale; MXFP4 1 or 4/3
    fmt: int
    mask: Optional[np.ndarray] = None  # (rows, cols) bool, QuEST: 1 = clipped
    extra: dict = field(default_factory=dict)

    @property
    def group(self):
        return GROUP[self.fmt]


# ------------------------------------------------------------ helpers ----
def abs_max(x):
    """Exact max |x| (order-free)."""
    x = np.asarray(x, dtype=F32)
    return F32(np.max(np.abs(x))) if x.size else F32(0.0)


def _groups(x, g):
    rows, cols = x.shape
    assert cols % g == 0, "cols must be a multiple of the group size"
    return x.reshape(rows, cols // g, g)


def _group_max(xg):
    return np.max(np.abs(xg), axis=-1).astype(F32)


def _encode_rtn(xg, d):
    """Codes of RTN_E2M1(x * fp32(1/d)) per group scale d (fp32).  A group
    whose reciprocal scale is not finite (d = 0, or d < 2^-128) encodes as
    zeros.  Returns (codes, v) with v the normalised values."""
    with np.errstate(divide="ignore", over="ignore", invalid="ignore"):
        inv = (F32(1.0) / d).astype(F32)
        ok = np.isfinite(inv) & (d > 0)
        inv = np.where(ok, inv, F32(0.0)).astype(F32)
        v = (xg * inv[..., None]).astype(F32)
    codes = fm.rtn_e2m1(v)
    codes = np.where(ok[..., None], codes, 0).astype(np.uint8)
    return codes, v, ok


def _sse(xg, codes, d):
    """Sum over the group of fp32((x - fp32(q * d))^2), pairwise tree."""
    q = fm.decode_e2m1(codes)
    deq = (q * d[..., None]).astype(F32)
    e = (xg - deq).astype(F32)
    return fm.pairwise_sum((e * e).astype(F32))


def _sr_index(rows, cols, row_ids=None):
    """Linear element indices (the Philox counter of element SR): rows are
    rows 0..rows-1 of the tensor, or the rows ``row_ids`` of a larger tensor
    with the same number of columns."""
    if row_ids is None:
        return np.arange(rows * cols, dtype=np.uint64).reshape(rows, cols)
    r = np.asarray(row_ids, dtype=np.uint64).reshape(rows, 1)
    return r * np.uint64(cols) + np.arange(cols, dtype=np.uint64)[None, :]


# ---------------------------------------------------------------- NVFP4 ----
def nvfp4_tensor_scale(amax, div):
    """x_fp32 = amax / div; a zero result (all-zero tensor) becomes 1.0."""
    s32 = F32(F32(amax) / div)
    return F32(1.0) if s32 == 0 else s32


def nvfp4_rtn(x, amax=None):
    """NVFP4 round-to-nearest with AbsMax scales (Quartet II page, MS-EDEN
    Step 2 with s = 6; the deterministic quantizer of the forward pass)."""
    x = np.asarray(x, dtype=F32)
    amax = abs_max(x) if amax is None else F32(amax)
    s32 = nvfp4_tensor_scale(amax, NV_RTN_DIV)
    xg = _groups(x, 16)
    gmax = _group_max(xg)
    s8 = fm.rtn_e4m3((gmax / F32(s32 * F32(6.0))).astype(F32))
    d = (fm.e4m3_value(s8).astype(F32) * s32).astype(F32)
    codes, _, _ = _encode_rtn(xg, d)
    return QTensor(codes.reshape(x.shape), s8, s32, NVFP4)


def nvfp4_rtn_square16(x, amax=None):
    """NVFP4 round-to-nearest with one E4M3 scale per 16 x 16 block (the
    square-block weight quantisation of the NVIDIA recipe, Quartet II page,
    "The square-block trade-off" and Table 1 "16x16"): the block maximum takes
    the place of the 1 x 16 group maximum in the RTN rule.  The scales are
    returned per 1 x 16 group (rows x cols/16, each block's scale repeated on
    its 16 rows), the layout the block-scaled GEMM reads.  Rows and columns
    are multiples of 16.  Quantising x^T gives the transpose of quantising x
    (the blocks and the rule are symmetric), which is what lets the recipe
    re-use Q(W) for W^T."""
    x = np.asarray(x, dtype=F32)
    rows, cols = x.shape
    assert rows % 16 == 0 and cols % 16 == 0, "16 x 16 blocks need rows and cols divisible by 16"
    amax = abs_max(x) if amax is None else F32(amax)
    s32 = nvfp4_tensor_scale(amax, NV_RTN_DIV)
    bmax = np.abs(x).reshape(rows // 16, 16, cols // 16, 16).max(axis=(1, 3)).astype(F32)
    sb = fm.rtn_e4m3((bmax / F32(s32 * F32(6.0))).astype(F32))
    s8 = np.repeat(sb, 16, axis=0)                       # rows x cols/16
    d = (fm.e4m3_value(s8).astype(F32) * s32).astype(F32)
    codes, _, _ = _encode_rtn(_groups(x, 16), d)
    return QTensor(codes.reshape(x.shape), s8.astype(np.uint8), s32, NVFP4)


def transpose_square16(qt):
    """The transpose of a 16 x 16 square-block quantised tensor: codes
    transposed, each block's scale moved to the transposed block (the
    re-use of Q(W) as Q(W^T) in the NVIDIA recipe's dX GEMM)."""
    rows, cols = qt.codes.shape
    assert qt.fmt == NVFP4 and rows % 16 == 0 and cols % 16 == 0
    sb = qt.scales[::16]                                  # block scales (rows/16 x cols/16)
    return QTensor(np.ascontiguousarray(qt.codes.T), np.repeat(sb.T, 16, axis=0).astype(np.uint8),
                   qt.tensor_scale, NVFP4)


def nvfp4_four_over_six(x, amax=None):
    """Four-Over-Six (Quartet II page, "Forward Pass Design", steps 1-4): per
    block of 16, quantise once with the block maximum mapped to 6 and once
    mapped to 4 (each scale rounded to E4M3), keep the one with the smaller
    squared error in the original domain.  READING: a tie keeps 6."""
    x = np.asarray(x, dtype=F32)
    amax = abs_max(x) if amax is None else F32(amax)
    s32 = nvfp4_tensor_scale(amax, NV_RTN_DIV)
    xg = _groups(x, 16)
    gmax = _group_max(xg)
    s8_6 = fm.rtn_e4m3((gmax / F32(s32 * F32(6.0))).astype(F32))
    s8_4 = fm.rtn_e4m3((gmax / F32(s32 * F32(4.0))).astype(F32))
    d6 = (fm.e4m3_value(s8_6).astype(F32) * s32).astype(F32)
    d4 = (fm.e4m3_value(s8_4).astype(F32) * s32).astype(F32)
    c6, _, _ = _encode_rtn(xg, d6)
    c4, _, _ = _encode_rtn(xg, d4)
    e6 = _sse(xg, c6, d6)
    e4 = _sse(xg, c4, d4)
    pick4 = e4 < e6
    codes = np.where(pick4[..., None], c4, c6)
    s8 = np.where(pick4, s8_4, s8_6).astype(np.uint8)
    return QTensor(codes.reshape(x.shape), s8, s32, NVFP4,
                   extra={"pick4": pick4})


def nvfp4_sr(x, seed, tensor_tag, amax=None, row_ids=None):
    """NVIDIA-style NVFP4 stochastic rounding (Quartet II page, "NVFP4 Format
    and Standard Stochastic Rounding", Steps 1-3): the 16/17 guard makes the
    normalised values stay within [-6, 6] so SR never clips."""
    x = np.asarray(x, dtype=F32)
    rows, cols = x.shape
    amax = abs_max(x) if amax is None else F32(amax)
    s32 = nvfp4_tensor_scale(amax, NV_SR_DIV)
    xg = _groups(x, 16)
    gmax = _group_max(xg)
    s8 = fm.rtn_e4m3((gmax / F32(s32 * NV_SR_GROUP_DIV)).astype(F32))
    d = (fm.e4m3_value(s8).astype(F32) * s32).astype(F32)
    _, v, ok = _encode_rtn(xg, d)
    u = philox.uniform(seed, _sr_index(rows, cols, row_ids), philox.TAG_SR_ELEM, tensor_tag)
    codes = fm.sr_e2m1(v.reshape(rows, cols), u)
    codes = np.where(ok.repeat(16, axis=-1), codes, 0).astype(np.uint8)
    return QTensor(codes, s8, s32, NVFP4)


def nvfp4_quest(x, amax=None):
    """QuEST RMSE-optimal clipping on NVFP4 (Quartet page, "The Forward-Pass
    Quantization: QuEST in Detail"), on the E4M3 scale grid.

    READINGS: sigma is the RMS of the group (the Hadamard output is centred;
    the FP4 grid has no zero point); the clip threshold of a scale d is
    T = 6 d; the search visits every E4M3 scale whose T satisfies
    sigma^2 <= T^2 <= 25 sigma^2 (c in [1, 5]), compared in fp32; ties keep the
    larger scale; an empty window falls back to the AbsMax rule.  The mask
    flags elements with |x / d| > 6 (clipped)."""
    x = np.asarray(x, dtype=F32)
    amax = abs_max(x) if amax is None else F32(amax)
    s32 = nvfp4_tensor_scale(amax, NV_RTN_DIV)
    xg = _groups(x, 16)
    gmax = _group_max(xg)
    sig2 = (fm.pairwise_sum((xg * xg).astype(F32)) / F32(16.0)).astype(F32)
    hi = (F32(25.0) * sig2).astype(F32)
    best_c = np.zeros(gmax.shape, dtype=np.int64)
    best_e = np.full(gmax.shape, np.inf, dtype=np.float64)
    found = np.zeros(gmax.shape, dtype=bool)
    for c in range(1, 127):                      # ascending scale
        d = (F32(fm.E4M3_VALUES[c]) * s32).astype(F32)
        t = F32(F32(6.0) * d)
        t2 = F32(t * t)
        inwin = (sig2 <= t2) & (t2 <= hi)
        if not inwin.any():
            continue
        dd = np.full(gmax.shape, d, dtype=F32)
        codes, _, _ = _encode_rtn(xg, dd)
        e = _sse(xg, codes, dd).astype(np.float64)
        better = inwin & (e <= best_e)           # <= : ties go to larger scale
        best_c = np.where(better, c, best_c)
        best_e = np.where(better, e, best_e)
        found |= inwin
    s8_fallback = fm.rtn_e4m3((gmax / F32(s32 * F32(6.0))).astype(F32)).astype(np.int64)
    s8 = np.where(found, best_c, s8_fallback).astype(np.uint8)
    d = (fm.e4m3_value(s8).astype(F32) * s32).astype(F32)
    codes, v, ok = _encode_rtn(xg, d)
    mask = (np.abs(v) > F32(6.0)) & ok[..., None]
    return QTensor(codes.reshape(x.shape), s8, s32, NVFP4,
                   mask=mask.reshape(x.shape))


def pairwise_sum_f64(v):
    """Sum of a 1-D array in float64 as a fixed pairwise tree over its order,
    padded with zeros to a power of two (the padding length does not change
    the value)."""
    a = np.asarray(v, dtype=np.float64).reshape(-1)
    n = 1
    while n < a.size:
        n <<= 1
    a = np.concatenate([a, np.zeros(n - a.size)])
    while a.size > 1:
        a = a[0::2] + a[1::2]
    return np.float64(a[0]) if a.size else np.float64(0.0)


def mse_group_scales(xg, s_T):
    """The group step of the MSE-optimal scale search ("Bridging the Gap
    Between Promise and Performance for Microscaling FP4 Quantization" page,
    "MSE-Optimized Grid and Scale Selection"): with the
    tensor scale s_T held, each 16-element group takes the E4M3 scale code c
    (1..126) whose RTN codes give the smallest squared error, the error of a
    candidate being the fp32 pairwise sum of fp32((x - fp32(q d))^2) with
    d = fp32(E4M3(c) s_T).  READINGS: the "1-D line search" visits every
    finite non-zero E4M3 code; ties keep the larger scale; a group whose
    maximum is zero takes code 0 (all codes zero), as under RTN."""
    gmax = _group_max(xg)
    best_c = np.zeros(gmax.shape, dtype=np.int64)
    best_e = np.full(gmax.shape, np.inf, dtype=F32)
    for c in range(1, 127):
        dd = np.full(gmax.shape, F32(F32(fm.E4M3_VALUES[c]) * F32(s_T)), dtype=F32)
        codes, _, _ = _encode_rtn(xg, dd)
        e = _sse(xg, codes, dd)
        better = e <= best_e                     # ascending scale: ties go to the larger
        best_c = np.where(better, c, best_c)
        best_e = np.where(better, e, best_e).astype(F32)
    return np.where(gmax > 0, best_c, 0).astype(np.uint8)


def mse_tensor_scale(x, s8, codes, s_T):
    """The tensor-scale step: with the group scale codes and the element codes
    held, the de-quantised tensor is s_T * u with u = E4M3(c_j) q_i, and the
    squared error is smallest at s_T = <x, u> / <u, u>.  READING: the page's
    second 1-D search is this closed-form least-squares solution; both inner
    products are float64 pairwise trees over the row-major element order
    (every product is exact in float64), the quotient is rounded once to
    fp32, and s_T is kept when either sum is not positive or the quotient is
    not a finite positive fp32 value."""
    u = (fm.e4m3_value(s8).astype(np.float64)[..., None]
         * fm.decode_e2m1(codes).astype(np.float64).reshape(s8.shape + (16,)))
    x64 = np.asarray(x, dtype=F32).astype(np.float64).reshape(u.shape)
    num = pairwise_sum_f64(x64 * u)
    den = pairwise_sum_f64(u * u)
    if not (num > 0 and den > 0):
        return F32(s_T)
    with np.errstate(over="ignore"):
        t = F32(num / den)
    return t if (np.isfinite(t) and t > 0) else F32(s_T)


def nvfp4_mse_search(x, iters):
    """NVFP4 with MSE-optimal scales by alternating optimisation ("Bridging
    the Gap Between Promise and Performance for Microscaling FP4 Quantization"
    page, "MSE-Optimized Grid and Scale Selection", NVFP4 without rotations):
    start from the RTN tensor scale amax / (6 * 256); a
    group step; then `iters` times a tensor-scale step followed by a group
    step.  The codes are RTN_E2M1(x * fp32(1/d)) at the final scales.  Each
    step lowers (or keeps) the exact squared error, so the error does not
    grow with `iters`.  Returns the QTensor and the tensor scale after each
    step in ``extra["s_T"]``."""
    x = np.asarray(x, dtype=F32)
    amax = abs_max(x)
    s_T = nvfp4_tensor_scale(amax, NV_RTN_DIV)
    xg = _groups(x, 16)
    history = [s_T]

    def group_step(s_T):
        s8 = mse_group_scales(xg, s_T)
        d = (fm.e4m3_value(s8).astype(F32) * F32(s_T)).astype(F32)
        codes, _, _ = _encode_rtn(xg, d)
        return s8, codes

    s8, codes = group_step(s_T)
    for _ in range(iters):
        s_T = mse_tensor_scale(x, s8, codes, s_T)
        history.append(s_T)
        s8, codes = group_step(s_T)
    return QTensor(codes.reshape(x.shape), s8, F32(s_T), NVFP4, extra={"s_T": history})


def ms_eden_pass1(y, chunk):
    """MS-EDEN first kernel of the post hoc range alignment (Quartet II page,
    "Post hoc range alignment kernel design"; Algorithm 1 Steps 2-3), on the
    already rotated y: per group of 16 an E8M3 pseudo-scale p = E8M3(gmax/s),
    RTN codes against p, per rotation chunk the EDEN factor
    S = <y, y> / <y, q p> (READING: a non-positive denominator gives S = 1),
    and the global max |y|."""
    y = np.asarray(y, dtype=F32)
    rows, cols = y.shape
    yg = _groups(y, 16)
    gmax = _group_max(yg)
    p = fm.e8m3_round((gmax / MS_EDEN_S).astype(F32))
    codes, _, ok = _encode_rtn(yg, p)
    xr = (fm.decode_e2m1(codes) * p[..., None]).astype(F32).reshape(rows, cols)
    yc = y.reshape(rows, cols // chunk, chunk)
    num = fm.pairwise_sum((yc * yc).astype(F32))
    den = fm.pairwise_sum((yc * xr.reshape(yc.shape)).astype(F32))
    with np.errstate(divide="ignore", invalid="ignore"):
        S = np.where(den > 0, (num / den).astype(F32), F32(1.0)).astype(F32)
    return codes.reshape(rows, cols), p, S, abs_max(y)


def ms_eden_tensor_scale(amax):
    """READING: the post hoc second kernel "shifts" the pseudo-scales into
    the FP8 range, so the tensor scale is the power of two
    x_fp32 = 2^k, k = ceil(log2(fp32(amax / (s * 256)))), the smallest power
    of two not below Algorithm 1's x_fp32 (largest shifted scale <= 256).
    p * 2^-k is then exact and the only FP8 rounding is the SR of S * p, as
    in Algorithm 1 Step 4 where SR acts on S times an on-grid FP8 scale.
    (Table 1's 9.8e-3 is reproduced this way, about 9.7e-3; a non power of two
    x_fp32 re-rounds p onto an unrelated grid and gives about 10.4e-3.)"""
    q = F32(F32(amax) / MS_EDEN_DIV)
    if q == 0:
        return F32(1.0)
    m, ex = np.frexp(float(q))          # q = m 2^ex, m in [0.5, 1)
    k = ex - 1 if m == 0.5 else ex
    return F32(np.ldexp(1.0, max(k, -126)))      # kept a normal fp32


def ms_eden_pass2(p, S, amax, chunk, seed, tensor_tag, row_ids=None):
    """MS-EDEN second kernel: shift the pseudo-scales into the FP8 range by
    the power-of-two tensor scale, fold in the EDEN factor S of their
    rotation chunk and round to E4M3 stochastically (Algorithm 1 Step 4; post
    hoc range alignment)."""
    rows, ng = p.shape
    s32 = ms_eden_tensor_scale(amax)
    inv32 = F32(F32(1.0) / s32)
    Sg = np.repeat(S, chunk // 16, axis=-1).astype(F32)
    t = ((Sg * p).astype(F32) * inv32).astype(F32)
    u = philox.uniform(seed, _sr_index(rows, ng, row_ids), philox.TAG_SR_SCALE, tensor_tag)
    s8 = fm.sr_e4m3(t, u)
    return s8, s32


def ms_eden_algorithm1(y, chunk, seed, tensor_tag):
    """Algorithm 1 of the Quartet II page taken literally (oracle-only
    statistical cross-check of the post hoc form): x_fp32 = amax/(s 256),
    E4M3 RTN group scales, RTN codes against them, S against the dequantised
    RTN tensor, then SR_FP8(S * x_fp8)."""
    y = np.asarray(y, dtype=F32)
    rows, cols = y.shape
    amax = abs_max(y)
    s32 = nvfp4_tensor_scale(amax, MS_EDEN_DIV)
    yg = _groups(y, 16)
    gmax = _group_max(yg)
    s8 = fm.rtn_e4m3((gmax / F32(s32 * MS_EDEN_S)).astype(F32))
    d = (fm.e4m3_value(s8).astype(F32) * s32).astype(F32)
    codes, _, _ = _encode_rtn(yg, d)
    xr = (fm.decode_e2m1(codes) * d[..., None]).astype(F32).reshape(rows, cols)
    yc = y.reshape(rows, cols // chunk, chunk)
    num = fm.pairwise_sum((yc * yc).astype(F32))
    den = fm.pairwise_sum((yc * xr.reshape(yc.shape)).astype(F32))
    with np.errstate(divide="ignore", invalid="ignore"):
        S = np.where(den > 0, (num / den).astype(F32), F32(1.0)).astype(F32)
    t = (np.repeat(S, chunk // 16, axis=-1) * fm.e4m3_value(s8).astype(F32)).astype(F32)
    u = philox.uniform(seed, np.arange(rows * (cols // 16), dtype=np.uint64).reshape(rows, -1),
                       philox.TAG_SR_SCALE, tensor_tag)
    return QTensor(codes.reshape(rows, cols), fm.sr_e4m3(t, u), s32, NVFP4)


def nvfp4_ms_eden(y, chunk, seed, tensor_tag, amax=None, row_ids=None):
    """Both passes; ``amax`` (the global max |y| of the whole tensor) and
    ``row_ids`` let a sample of the tensor's rows be quantised alone."""
    codes, p, S, amax1 = ms_eden_pass1(y, chunk)
    amax = amax1 if amax is None else F32(amax)
    s8, s32 = ms_eden_pass2(p, S, amax, chunk, seed, tensor_tag, row_ids)
    return QTensor(codes, s8, s32, NVFP4, extra={"pseudo": p, "S": S, "amax": amax})


# ---------------------------------------------------------------- MXFP4 ----
def mx_exponent(gmax):
    """READING (OCP MX rule): e = floor(log2 gmax) - 2, clamped to
    [-127, 127]; gmax = 0 gives -127.  The largest normalised magnitude then
    lies in [4, 8) and RTN saturates values above 6."""
    gmax = np.asarray(gmax, dtype=F32)
    _, ex = np.frexp(gmax.astype(np.float64))
    e = np.where(gmax > 0, ex - 1 - 2, -127)
    return np.clip(e, -127, 127).astype(np.int64)


def _pow2_f32(e):
    return np.ldexp(F32(1.0), np.asarray(e, dtype=np.int64)).astype(F32)


def _encode_pow2(xg, e):
    v = (xg * _pow2_f32(-e)[..., None]).astype(F32)
    return fm.rtn_e2m1(v), v


def mxfp4_rtn(x):
    """MXFP4 RTN with AbsMax (E8M0) scales (Quartet page, forward-pass
    candidates; Bridging-the-Gap page, MXFP4 format)."""
    x = np.asarray(x, dtype=F32)
    xg = _groups(x, 32)
    e = mx_exponent(_group_max(xg))
    codes, _ = _encode_pow2(xg, e)
    return QTensor(codes.reshape(x.shape), (e + 127).astype(np.uint8), F32(1.0), MXFP4)


def mxfp4_sr(x, seed, tensor_tag, row_ids=None):
    """Quartet backward quantizer G_q = SR(3/4 G_h) on MXFP4 (Quartet page,
    "Backward-Pass Quantization", the 3/4 rescaling factor).  READING: the
    exponent comes from the unscaled group max (OCP rule) and the values are
    multiplied by 3/4, so the largest normalised value lies in [3, 6) and SR
    never clips; the 4/3 is carried as the tensor scale, giving the 16/9
    after the GEMM."""
    x = np.asarray(x, dtype=F32)
    rows, cols = x.shape
    xg = _groups(x, 32)
    e = mx_exponent(_group_max(xg))
    v = ((xg * QUARTET_PRESCALE).astype(F32) * _pow2_f32(-e)[..., None]).astype(F32)
    u = philox.uniform(seed, _sr_index(rows, cols, row_ids), philox.TAG_SR_ELEM, tensor_tag)
    codes = fm.sr_e2m1(v.reshape(rows, cols), u)
    return QTensor(codes, (e + 127).astype(np.uint8), QUARTET_TENSOR_SCALE, MXFP4)


def mxfp4_quest(x):
    """QuEST on MXFP4 (Quartet page, "QuEST in Detail"): the same READINGS as
    ``nvfp4_quest`` on the power-of-two scale grid 2^e."""
    x = np.asarray(x, dtype=F32)
    xg = _groups(x, 32)
    gmax = _group_max(xg)
    sig2 = (fm.pairwise_sum((xg * xg).astype(F32)) / F32(32.0)).astype(F32)
    hi = (F32(25.0) * sig2).astype(F32)
    _, ex = np.frexp(sig2.astype(np.float64))
    fl = np.where(sig2 > 0, ex - 1, -300)                 # floor(log2 sigma^2)
    e_lo = np.floor_divide(fl, 2) - 4
    best_e = np.zeros(gmax.shape, dtype=np.int64)
    best_s = np.full(gmax.shape, np.inf, dtype=np.float64)
    found = np.zeros(gmax.shape, dtype=bool)
    for k in range(8):                                   # ascending scale
        e = np.clip(e_lo + k, -127, 125)
        t = (F32(6.0) * _pow2_f32(e)).astype(F32)
        t2 = (t * t).astype(F32)
        inwin = (sig2 <= t2) & (t2 <= hi) & (sig2 > 0)
        codes, _ = _encode_pow2(xg, e)
        d = _pow2_f32(e)
        s = _sse(xg, codes, d).astype(np.float64)
        better = inwin & (s <= best_s)
        best_e = np.where(better, e, best_e)
        best_s = np.where(better, s, best_s)
        found |= inwin
    e = np.where(found, best_e, mx_exponent(gmax))
    codes, v = _encode_pow2(xg, e)
    mask = np.abs(v) > F32(6.0)
    return QTensor(codes.reshape(x.shape), (e + 127).astype(np.uint8), F32(1.0), MXFP4,
                   mask=mask.reshape(x.shape))


# ------------------------------------------------------------ dispatch ----
def supported(fmt, rnd, had_block):
    """Combinations the pages define.  Four-Over-Six and MS-EDEN are NVFP4
    methods on the Quartet II page; MS-EDEN needs a rotation (its S lives on
    rotation groups) whose blocks contain whole scale groups."""
    if had_block not in (0, 16, 32, 64, 128, 256):
        return False
    if fmt == MXFP4 and rnd in (FOUR_OVER_SIX, MS_EDEN):
        return False
    if rnd == MS_EDEN and (had_block == 0 or had_block < GROUP[fmt]):
        return False
    if rnd == RTN_SQUARE16 and (fmt != NVFP4 or had_block != 0):
        return False
    return True


def quantize_transformed(y, fmt, rnd, seed=0, tensor_tag=0, chunk=None, amax=None, row_ids=None):
    """Quantise an already transformed fp32 tensor (groups along cols).  For
    a sample of a larger tensor's rows: ``amax`` is the whole tensor's max
    |y| (NVFP4 tensor scale) and ``row_ids`` its row indices (Philox
    counters); every other step is row-local."""
    if fmt == NVFP4:
        if rnd == RTN:
            return nvfp4_rtn(y, amax)
        if rnd == FOUR_OVER_SIX:
            return nvfp4_four_over_six(y, amax)
        if rnd == SR:
            return nvfp4_sr(y, seed, tensor_tag, amax, row_ids)
        if rnd == QUEST:
            return nvfp4_quest(y, amax)
        if rnd == MS_EDEN:
            return nvfp4_ms_eden(y, chunk, seed, tensor_tag, amax, row_ids)
        if rnd == RTN_SQUARE16:
            return nvfp4_rtn_square16(y, amax)
    else:
        if rnd == RTN:
            return mxfp4_rtn(y)
        if rnd == SR:
            return mxfp4_sr(y, seed, tensor_tag, row_ids)
        if rnd == QUEST:
            return mxfp4_quest(y)
    raise ValueError("unsupported format / rounding combination")


def quantize(x, fmt, rnd, had_block=0, randomized=False, seed=0, sign_tag=0,
             tensor_tag=0, transpose=False):
    """The whole quantizer: optional transpose (the quantised tensor is x^T,
    so the groups run along x's rows), the block (randomized) Hadamard along
    the inner dimension, then the chosen format and rounding."""
    if not supported(fmt, rnd, had_block):
        raise ValueError("unsupported format / rounding / Hadamard combination")
    a = np.asarray(x, dtype=F32)
    if transpose:
        a = np.ascontiguousarray(a.T)
    y = hd.block_transform(a, had_block, randomized, seed, sign_tag)
    return quantize_transformed(y, fmt, rnd, seed, tensor_tag, chunk=had_block)


def transformed_abs_max(x, had_block=0, randomized=False, seed=0, sign_tag=0, transpose=False,
                        rows_per_chunk=2048):
    """max |y| of the whole transformed tensor y = block_transform(x or x^T),
    computed a chunk of rows at a time (the rotation is row-local)."""
    a = np.asarray(x).T if transpose else np.asarray(x)
    m = F32(0.0)
    for r0 in range(0, a.shape[0], rows_per_chunk):
        y = hd.block_transform(np.ascontiguousarray(a[r0:r0 + rows_per_chunk], dtype=F32), had_block,
                               randomized, seed, sign_tag)
        m = max(m, abs_max(y))
    return F32(m)


def quantize_rows(x, rows, fmt, rnd, had_block=0, randomized=False, seed=0, sign_tag=0,
                  tensor_tag=0, transpose=False, amax=None):
    """Rows ``rows`` of ``quantize(x, ...)`` (codes, scales, tensor scale),
    from those rows of the (transposed) input alone: rotation, scales and
    codes are row-local; NVFP4 also needs the whole transformed tensor's
    max |y| (``amax``, computed here when not given) and the stochastic modes
    index Philox by the rows' positions in the whole tensor."""
    if not supported(fmt, rnd, had_block):
        raise ValueError("unsupported format / rounding / Hadamard combination")
    rows = np.asarray(rows, dtype=np.int64)
    a = np.asarray(x).T if transpose else np.asarray(x)
    sub = np.ascontiguousarray(a[rows], dtype=F32)
    y = hd.block_transform(sub, had_block, randomized, seed, sign_tag)
    if fmt == NVFP4 and amax is None:
        amax = transformed_abs_max(x, had_block, randomized, seed, sign_tag, transpose)
    return quantize_transformed(y, fmt, rnd, seed, tensor_tag, chunk=had_block, amax=amax, row_ids=rows)


# ------------------------------------------------------- dequantisation ----
def scale_values(qt):
    if qt.fmt == MXFP4:
        return fm.e8m0_value(qt.scales)
    return fm.e4m3_value(qt.scales)


def dequant_f32(qt):
    """fp32 dequantisation as the re-quantisation step reads a saved tensor:
    fp32(fp32(q * s_group) * s_tensor) (q * s_group is exact)."""
    g = qt.group
    rows, cols = qt.codes.shape
    q = fm.decode_e2m1(qt.codes).reshape(rows, cols // g, g)
    s = scale_values(qt).astype(F32)
    v = (q * s[..., None]).astype(F32)
    v = (v * F32(qt.tensor_scale)).astype(F32)
    return v.reshape(rows, cols)


def dequant_f64(qt, with_tensor_scale=True):
    """Exact fp64 value of every element: q * s_group (* s_tensor)."""
    g = qt.group
    rows, cols = qt.codes.shape
    q = fm.decode_e2m1(qt.codes).astype(np.float64).reshape(rows, cols // g, g)
    v = (q * scale_values(qt)[..., None]).reshape(rows, cols)
    if with_tensor_scale:
        v = v * float(qt.tensor_scale)
    return v


def requantize(qt, rnd, had_block=0, randomized=False, seed=0, sign_tag=0,
               tensor_tag=0, transpose=True, fmt=None):
    """Quartet II page, "The Complete Quartet II Computation Graph", backward
    steps 1-4: de-quantise a saved tensor, transpose it, rotate along the new
    inner dimension and quantise again."""
    fmt = qt.fmt if fmt is None else fmt
    return quantize(dequant_f32(qt), fmt, rnd, had_block, randomized, seed,
                    sign_tag, tensor_tag, transpose)


# ------------------------------------------------- tensor-core layout ----
def swizzled_scale_shape(rows, n_groups):
    """Bytes of the tensor-core scale layout: 128-row x 4-group atoms of 512
    bytes, rows padded to 128 and groups to 4 (zero filled)."""
    return (rows + 127) // 128, (n_groups + 3) // 4


def swizzle_scales(scales):
    """Linear (rows, n_groups) scales -> the tensor-core block-scale layout:
    byte (r, k) goes to ((r//128) * nkb + k//4) * 512 + (r%32) * 16
    + ((r%128)//32) * 4 + k%4.  Padding is zero."""
    rows, ng = scales.shape
    nrb, nkb = swizzled_scale_shape(rows, ng)
    out = np.zeros(nrb * nkb * 512, dtype=np.uint8)
    r = np.arange(rows)[:, None]
    k = np.arange(ng)[None, :]
    off = ((r // 128) * nkb + k // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + k % 4
    out[off.reshape(-1)] = scales.reshape(-1)
    return out


# ----------------------------------------------------- MXFP4 scale fit ----
@dataclass
class FitTensor:
    """MXFP4 with fitted fractional-exponent scales (MXFP4-dagger): E2M1
    codes, one 8-bit level q per 32-element group and the tensor's table of
    the 256 scale values 2^(alpha q + beta)."""
    codes: np.ndarray          # (rows, cols) uint8
    q: np.ndarray              # (rows, cols // 32) uint8
    table: np.ndarray          # (256,) float32
    thresholds: np.ndarray     # (255,) float32, level k -> k + 1 boundary
    l_min: float
    alpha: float


def mxfp4_fit_levels(s_min, s_max):
    """Bridging-the-Gap page, "MXFP Scale Fitting" (Appendix H, the
    MXFP4-dagger remap): with L = log2 of the smallest and largest group
    scale of the tensor, level q in [0, 255] stands for the scale
    2^(alpha q + L_min), alpha = (L_max - L_min) / 255 -- a fractional
    exponent step (READING: the printed formula is garbled, it multiplies the
    level by L_max - L_min; the page's own summary s = 2^(alpha q + beta) with
    alpha in (0, 1) fixes the 1/255).  Level k and k + 1 meet where the
    log-scale crosses alpha (k + 0.5), the page's round().  Returns the fp32
    table of the 256 scales, the 255 fp32 boundaries, L_min and alpha; every
    exponent is computed in fp64 and rounded once to fp32."""
    l_min = float(np.log2(np.float64(s_min)))
    l_max = float(np.log2(np.float64(s_max)))
    alpha = (l_max - l_min) / 255.0
    q = np.arange(256, dtype=np.float64)
    table = np.exp2(l_min + alpha * q).astype(F32)
    thr = np.exp2(l_min + alpha * (q[:255] + 0.5)).astype(F32)
    return table, thr, l_min, alpha


def mxfp4_fit(x):
    """MXFP4-dagger quantisation of an (already transformed) fp32 tensor,
    RTN elements.  READINGS: the group scale before fitting is the AbsMax
    scale s = fp32(gmax / 6) (the modified formula drops the 4/3 bias of the
    original rule); L_min and L_max come from the groups with s > 0; a
    group's level is the number of boundaries t_k with s >= t_k (the
    round() of the page, ties up); the elements are RTN_E2M1(x * fp32(1/d))
    with d = table[q], saturating at 6, as the other RTN rules here; a group
    with s = 0, or whose reciprocal scale is not finite, encodes as zeros
    with level 0; a tensor with no s > 0 gets the table of s = 1; when every
    s > 0 is equal, alpha = 0, all levels and boundaries equal s and the
    count gives level 255.
    (The E8M0 block scaling of the tensor cores cannot apply these scales:
    they are not powers of two.)"""
    x = np.asarray(x, dtype=F32)
    rows, cols = x.shape
    xg = _groups(x, 32)
    s = (_group_max(xg) / F32(6.0)).astype(F32)
    pos = s > 0
    if pos.any():
        table, thr, l_min, alpha = mxfp4_fit_levels(s[pos].min(), s[pos].max())
    else:
        table, thr, l_min, alpha = mxfp4_fit_levels(F32(1.0), F32(1.0))
    q = (s[..., None] >= thr).sum(axis=-1).astype(np.int64)
    q = np.where(pos, q, 0)
    d = table[q]
    with np.errstate(divide="ignore", over="ignore"):
        inv = (F32(1.0) / d).astype(F32)
    ok = pos & np.isfinite(inv)
    v = (xg * np.where(ok, inv, F32(0.0))[..., None]).astype(F32)
    codes = fm.rtn_e2m1(v).reshape(rows, cols)
    return FitTensor(codes, q.astype(np.uint8), table, thr, l_min, alpha)


def mxfp4_fit_dequant(ft):
    """fp32(code * table[q]) per element (q * d is exact: one significant
    bit pair times an fp32 scale)."""
    rows, cols = ft.codes.shape
    q = fm.decode_e2m1(ft.codes).reshape(rows, cols // 32, 32)
    d = ft.table[ft.q.astype(np.int64)]
    return (q * d[..., None]).astype(F32).reshape(rows, cols)
