"""GPU de-quantisation and the method diagnostics computed with the CUDA
path: de-quantised values bit-exact against the oracle's, the Quartet II
page's Table 1 MSEs reproduced from GPU-quantised tensors (and equal to the
oracle's on the same input), and the projection magnitude misalignment zero
for stochastic rounding (the Quartet page prints 0.00) and not for RTN."""
import numpy as np
import pytest
import torch

from fp4_microscaled_quantized_b200 import synthetic as syn
from oracle import hadamard as hd
from oracle import quant as qn

pytestmark = pytest.mark.gpu


def to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("fmt,rnd,had", [(qn.NVFP4, qn.FOUR_OVER_SIX, 0), (qn.NVFP4, qn.MS_EDEN, 128),
                                         (qn.NVFP4, qn.SR, 16), (qn.MXFP4, qn.QUEST, 32),
                                         (qn.MXFP4, qn.SR, 32), (qn.MXFP4, qn.RTN, 0)])
def test_dequantize_bit_exact(cuda_lib, fmt, rnd, had):
    bits = syn.outlier_elements((192, 512), seed=9, stream=rnd)
    x = syn.bf16_bits_to_f32(bits)
    g = cuda_lib.quantize(to_dev(bits), fmt, rnd, had, randomized=had > 0, seed=77, sign_tag=1, tensor_tag=2)
    o = qn.quantize(x, fmt, rnd, had, had > 0, 77, 1, 2)
    ref = qn.dequant_f32(o)
    d32 = cuda_lib.dequantize(g).cpu().numpy()
    np.testing.assert_array_equal(d32.view(np.uint32), ref.view(np.uint32))
    d16 = cuda_lib.dequantize(g, out_dtype=torch.bfloat16).cpu().view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(d16, syn.f32_to_bf16_bits(ref))


def test_dequantize_empty_and_errors(cuda_lib):
    q = cuda_lib.alloc_qtensor(0, 64, qn.NVFP4)
    assert cuda_lib.dequantize(q).shape == (0, 64)
    q = cuda_lib.alloc_qtensor(16, 64, qn.NVFP4, linear=False)
    with pytest.raises(cuda_lib.Fp4Error):
        cuda_lib.dequantize(q)                    # no linear scales


def test_table1_from_gpu_quantisers(cuda_lib):
    from fp4_microscaled_quantized_b200 import diagnostics as dg
    bits = syn.gaussian((1024, 1024), 1.0, 0)
    x = syn.bf16_bits_to_f32(bits)
    for rnd, had, page, rel in ((qn.RTN, 0, 9.0, 0.03), (qn.FOUR_OVER_SIX, 0, 7.6, 0.03),
                                (qn.SR, 0, 23.5, 0.03), (qn.MS_EDEN, 128, 9.8, 0.05),
                                (qn.RTN_SQUARE16, 0, 12.4, 0.03)):
        gpu = dg.quant_mse(qn.NVFP4, rnd, had, n_seeds=1)
        assert gpu == pytest.approx(page, rel=rel)
        # the same value from the oracle's quantisation of the same input
        rand = had > 0 or rnd == qn.SR
        y = hd.block_transform(x, had, rand, 0, 0) if had else x
        o = qn.quantize(x, qn.NVFP4, rnd, had, rand, 0, 0, 1)
        ora = 1e3 * float(np.mean((qn.dequant_f32(o).astype(np.float64) - y.astype(np.float64)) ** 2))
        assert gpu == pytest.approx(ora, rel=1e-6)


def test_misalignment_sr_zero_rtn_not(cuda_lib):
    from fp4_microscaled_quantized_b200 import diagnostics as dg
    m_sr, se_sr = dg.misalignment(qn.MXFP4, qn.SR, 32, n_seeds=32)
    m_rtn, se_rtn = dg.misalignment(qn.MXFP4, qn.RTN, 32, n_seeds=32)
    m_eden, se_eden = dg.misalignment(qn.NVFP4, qn.MS_EDEN, 128, n_seeds=32)
    assert abs(m_sr) < 4 * se_sr + 1e-6
    assert abs(m_eden) < 4 * se_eden + 3e-3          # MS-EDEN: unbiased to ~1e-3 (oracle pins)
    assert abs(m_rtn) > 10 * se_rtn


def test_mean_converges_like_one_over_B(cuda_lib):
    """Figure 9 of the Quartet II page from the CUDA path: the mean of B
    back-rotated MS-EDEN (and SR) samples approaches the input with an error
    falling like 1/B; RTN after a random rotation levels off."""
    from fp4_microscaled_quantized_b200 import diagnostics as dg
    Bs = (10, 100, 1000)
    eden = dg.mean_convergence(qn.NVFP4, qn.MS_EDEN, 128, n=1000, Bs=Bs)
    sr = dg.mean_convergence(qn.NVFP4, qn.SR, 128, n=1000, Bs=Bs)
    rtn = dg.mean_convergence(qn.NVFP4, qn.RTN, 128, n=1000, Bs=Bs)
    assert eden["slope"] <= -0.8 and sr["slope"] <= -0.8
    assert rtn["slope"] > -0.8
    assert eden["rel_sq_err"][-1] < rtn["rel_sq_err"][-1]
