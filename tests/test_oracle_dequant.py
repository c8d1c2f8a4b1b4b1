"""Pins of the oracle's fp32 de-quantisation, the input of every
re-quantisation (the backward operands Q(W)^T and Q(X)^T of every recipe).

Quartet II page, "NVFP4 Format and Standard Stochastic Rounding": a stored
element is x = x_fp4 * x_fp8 * x_fp32.  The oracle evaluates it in fp32 as
fp32(fp32(q * s_group) * s_tensor).  The inner product q * s_group is exact
in fp32 (q has at most two significant bits, an E4M3 scale at most four, an
E8M0 scale one), so the result must be the exact value q * s_group *
s_tensor rounded once to fp32, for every tensor scale the formats take:
any fp32 value for NVFP4 (q * s_group <= 6 * 448 never overflows), 1 or 4/3
for MXFP4 (Quartet's 3/4 pre-scale; a tensor scale >= 1 overflows exactly
when the exact value does).  An MXFP4 tensor scale below 1 with an E8M0
scale near 2^127 would overflow in q * s_group while the exact value is
finite; no quantiser here produces one, and test_dequant_f32_mxfp4_domain
shows the boundary.  These tests check the equality over every (code,
scale) pair of both formats, against the exact fp64 product, so a double
rounding (q * fp32(s_group * s_tensor)), a dropped factor or a wrong operand
would fail."""
import numpy as np

from oracle import formats as fm
from oracle import quant as qn

F32 = np.float32


def all_pairs(fmt):
    """A QTensor with one group per scale code and every E2M1 code in each
    group (codes 0..15, repeated to fill a 32-element MXFP4 group)."""
    g = qn.GROUP[fmt]
    n_scales = 127 if fmt == qn.NVFP4 else 255         # E4M3 0x7F and E8M0 0xFF are NaN
    codes = np.tile(np.arange(16, dtype=np.uint8), (n_scales, g // 16))
    scales = np.arange(n_scales, dtype=np.uint8)[:, None]
    return codes, scales


TENSOR_SCALES = {
    qn.NVFP4: [1.0, 2.0 ** -20, float(F32(1.0) / F32(3.0)), float(F32(37.25) / qn.NV_RTN_DIV),
               2.0 ** -140, float(F32(3.0e38) / F32(2688.0)), float(F32(1.0e-3) / qn.MS_EDEN_DIV)],
    qn.MXFP4: [1.0, float(qn.QUARTET_TENSOR_SCALE)],
}


def exact_f32(qt):
    """The exact value q * s_group * s_tensor (fp64 holds it: at most
    2 + 4 + 24 significant bits), rounded once to fp32."""
    with np.errstate(over="ignore"):
        return qn.dequant_f64(qt).astype(F32)


def test_dequant_f32_every_code_and_scale():
    for fmt in (qn.NVFP4, qn.MXFP4):
        codes, scales = all_pairs(fmt)
        for ts in TENSOR_SCALES[fmt]:
            qt = qn.QTensor(codes, scales, F32(ts), fmt)
            with np.errstate(over="ignore"):
                got = qn.dequant_f32(qt)
            want = exact_f32(qt)
            np.testing.assert_array_equal(fm.f32_bits(got), fm.f32_bits(want),
                                          err_msg="fmt %d tensor scale %r" % (fmt, ts))


def test_dequant_f32_covers_the_edges():
    """The pairs above reach fp32 subnormals, overflow to inf and -0."""
    codes, scales = all_pairs(qn.MXFP4)
    with np.errstate(over="ignore"):
        v = qn.dequant_f32(qn.QTensor(codes, scales, F32(1.0), qn.MXFP4))
    assert np.isinf(v).any()                               # 6 * 2^127 overflows
    tiny = v[(v != 0) & np.isfinite(v)]
    assert (np.abs(tiny) < np.finfo(F32).tiny).any()        # 0.5 * 2^-127 is subnormal
    assert (np.signbit(v) & (v == 0)).any()                 # code 8 is -0
    codes, scales = all_pairs(qn.NVFP4)
    v = qn.dequant_f32(qn.QTensor(codes, scales, F32(2.0 ** -140), qn.NVFP4))
    assert (np.abs(v[v != 0]) < np.finfo(F32).tiny).all()   # every non-zero product is subnormal


def test_dequant_f32_worked_values():
    """Values worked out by hand from the format definitions.
    NVFP4: E2M1 code 0b0111 = 6, E4M3 code 0x7E = 448, s_T = 2^-10:
    6 * 448 / 1024 = 2.625.  E2M1 0b1101 = -3, E4M3 0x01 = 2^-9 (the smallest
    subnormal), s_T = 1: -3 / 512.  E2M1 0b0001 = 0.5, E4M3 0x38 = 1.0,
    s_T = fp32(1/3) = 0x3EAAAAAB: 0.5 * fp32(1/3) = 0x3E2AAAAB.
    MXFP4: E2M1 0b0011 = 1.5, E8M0 130 = 2^3, s_T = fp32(4/3): 12 * fp32(4/3)
    = 16.000000477 rounds to 16.0 (half an ulp at 16 is 9.5e-7)."""
    def one(code, scale, ts, fmt):
        g = qn.GROUP[fmt]
        c = np.zeros((1, g), dtype=np.uint8)
        c[0, 0] = code
        return float(qn.dequant_f32(qn.QTensor(c, np.array([[scale]], dtype=np.uint8), F32(ts), fmt))[0, 0])

    assert one(0b0111, 0x7E, 2.0 ** -10, qn.NVFP4) == 2.625
    assert one(0b1101, 0x01, 1.0, qn.NVFP4) == -3.0 / 512.0
    third = F32(1.0) / F32(3.0)
    assert fm.f32_bits(third) == 0x3EAAAAAB
    assert fm.f32_bits(F32(one(0b0001, 0x38, third, qn.NVFP4))) == 0x3E2AAAAB
    assert one(0b0011, 130, qn.QUARTET_TENSOR_SCALE, qn.MXFP4) == 16.0


def test_dequant_f32_mxfp4_domain():
    """Outside the MXFP4 domain (a tensor scale below 1) the fp32 evaluation
    overflows early: 2 * 2^127 is inf in fp32, while 2 * 2^127 * 0.75 is
    finite.  Inside it the two agree (the test above)."""
    c = np.zeros((1, 32), dtype=np.uint8)
    c[0, 0] = 0b0100                                   # 2.0
    qt = qn.QTensor(c, np.array([[254]], dtype=np.uint8), F32(0.75), qn.MXFP4)
    with np.errstate(over="ignore"):
        assert np.isinf(qn.dequant_f32(qt)[0, 0])
    assert np.isfinite(exact_f32(qt)[0, 0])
