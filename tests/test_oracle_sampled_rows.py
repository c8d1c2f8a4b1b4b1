"""The oracle's sampled-rows path (used by the full-size GPU parity tests)
gives exactly the rows of the whole-tensor quantisation, in every mode: the
rotation, scales and codes are row-local, the NVFP4 tensor scale comes from
the whole tensor's max |y|, and the stochastic modes index Philox by the
row's position in the whole tensor."""
import numpy as np
import pytest

from fp4_microscaled_quantized_b200 import synthetic as syn
from oracle import quant as qn

CASES = [(qn.NVFP4, qn.RTN, 0), (qn.NVFP4, qn.FOUR_OVER_SIX, 16), (qn.NVFP4, qn.SR, 32),
         (qn.NVFP4, qn.QUEST, 0), (qn.NVFP4, qn.MS_EDEN, 128), (qn.MXFP4, qn.RTN, 32),
         (qn.MXFP4, qn.SR, 128), (qn.MXFP4, qn.QUEST, 32)]


@pytest.mark.parametrize("fmt,rnd,had", CASES)
@pytest.mark.parametrize("transpose", [False, True])
def test_quantize_rows_equals_whole_tensor_rows(fmt, rnd, had, transpose):
    x = syn.bf16_bits_to_f32(syn.outlier_elements((256, 384), seed=31, stream=rnd))
    full = qn.quantize(x, fmt, rnd, had, randomized=had > 0, seed=7, sign_tag=1, tensor_tag=4,
                       transpose=transpose)
    rows = np.array([0, 5, 77, 128, full.codes.shape[0] - 1])
    part = qn.quantize_rows(x, rows, fmt, rnd, had, randomized=had > 0, seed=7, sign_tag=1,
                            tensor_tag=4, transpose=transpose)
    np.testing.assert_array_equal(part.codes, full.codes[rows])
    np.testing.assert_array_equal(part.scales, full.scales[rows])
    assert np.float32(part.tensor_scale) == np.float32(full.tensor_scale)
    if full.mask is not None:
        np.testing.assert_array_equal(part.mask, full.mask[rows])
