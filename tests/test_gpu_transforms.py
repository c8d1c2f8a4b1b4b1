"""GPU parity of the Bridging-the-Gap page's forward-only variants against
the oracle, bit for bit: the DCT-II / DST-II block transforms (fp32 output),
every format and rounding mode quantising their output (fp4_quantize_f32),
and the MXFP4 scale fit (codes, levels, the 256-entry table, the
de-quantised values)."""
import numpy as np
import pytest
import torch

from fp4_microscaled_quantized_b200 import synthetic as syn
from oracle import formats as fm
from oracle import hadamard as hd
from oracle import quant as qn
from oracle import transforms as tr

pytestmark = pytest.mark.gpu

KIND = {"dct2": 1, "dst2": 2}


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("kind", tr.KINDS)
@pytest.mark.parametrize("k", [16, 32, 64, 128, 256])
def test_block_transform_bit_exact(cuda_lib, kind, k):
    """200 rows (a ragged last row tile), 2 blocks per row."""
    bits = syn.outlier_elements((200, 2 * k), seed=k, stream=KIND[kind])
    y = cuda_lib.block_transform(dev(bits), KIND[kind], k)
    want = tr.block_transform_f32(syn.bf16_bits_to_f32(bits), kind, k)
    np.testing.assert_array_equal(y.cpu().numpy().view(np.uint32), want.view(np.uint32))
    assert cuda_lib.get_last_error() == 0


@pytest.mark.parametrize("fmt,rnd", [(qn.NVFP4, qn.RTN), (qn.NVFP4, qn.QUEST), (qn.NVFP4, qn.FOUR_OVER_SIX),
                                     (qn.NVFP4, qn.SR), (qn.MXFP4, qn.RTN), (qn.MXFP4, qn.QUEST),
                                     (qn.MXFP4, qn.SR)])
@pytest.mark.parametrize("kind,k", [("dct2", 32), ("dst2", 128)])
def test_transform_then_quantize(cuda_lib, fmt, rnd, kind, k):
    bits = syn.student_t((136, 512), seed=11, unit_rms=True)
    y = cuda_lib.block_transform(dev(bits), KIND[kind], k)
    g = cuda_lib.quantize_f32(y, fmt, rnd, seed=0xABCDEF, tensor_tag=3)
    torch.cuda.synchronize()
    o = qn.quantize_transformed(tr.block_transform_f32(syn.bf16_bits_to_f32(bits), kind, k), fmt, rnd,
                                0xABCDEF, 3)
    np.testing.assert_array_equal(g.codes.cpu().numpy(), fm.pack_codes(o.codes))
    np.testing.assert_array_equal(g.scales.cpu().numpy(), o.scales)
    np.testing.assert_array_equal(g.scales_swz.cpu().numpy(), qn.swizzle_scales(o.scales))
    assert g.tensor_scale.cpu().numpy().view(np.uint32)[0] == np.float32(o.tensor_scale).view(np.uint32)
    if o.mask is not None:
        np.testing.assert_array_equal(g.mask.cpu().numpy(), fm.pack_mask(o.mask))
    assert cuda_lib.get_last_error() == 0


def test_quantize_f32_rejects_what_needs_its_own_input(cuda_lib):
    y = torch.zeros((64, 256), dtype=torch.float32, device="cuda")
    for rnd in (qn.MS_EDEN, qn.RTN_SQUARE16):
        with pytest.raises(cuda_lib.Fp4Error) as e:
            cuda_lib.quantize_f32(y, qn.NVFP4, rnd)
        assert e.value.status == 2                           # FP4_ERR_UNSUPPORTED


def _mixed(rows, cols, seed):
    """Gaussian rows with per-row scales over 2^-8 .. 2^8, rounded to bf16."""
    g = syn.gaussian((rows, cols), 1.0, seed=seed)
    sc = np.exp2(np.linspace(-8, 8, rows)).astype(np.float32)[:, None]
    return syn.f32_to_bf16_bits(syn.bf16_bits_to_f32(g) * sc)


@pytest.mark.parametrize("had", [0, 32, 128])
def test_mx_fit_bit_exact(cuda_lib, had):
    bits = _mixed(200, 512, seed=had + 1)
    ft = cuda_lib.quantize_mx_fit(dev(bits), had)
    d = cuda_lib.dequantize_mx_fit(ft)
    torch.cuda.synchronize()
    x = syn.bf16_bits_to_f32(bits)
    o = qn.mxfp4_fit(hd.block_transform(x, had, False) if had else x)
    np.testing.assert_array_equal(ft.table.cpu().numpy().view(np.uint32), o.table.view(np.uint32))
    np.testing.assert_array_equal(ft.levels.cpu().numpy(), o.q)
    np.testing.assert_array_equal(ft.codes.cpu().numpy(), fm.pack_codes(o.codes))
    np.testing.assert_array_equal(d.cpu().numpy().view(np.uint32), qn.mxfp4_fit_dequant(o).view(np.uint32))
    assert cuda_lib.get_last_error() == 0


def test_mx_fit_degenerate_inputs(cuda_lib):
    """A zero group, an all-zero tensor, one shared scale (alpha = 0), and
    two calls in a row on the same workspace."""
    bits = _mixed(64, 256, seed=5)
    bits[3, 64:96] = 0
    ws = cuda_lib.alloc_workspace(4096)
    for b in (bits, np.zeros((32, 128), dtype=np.uint16)):
        ft = cuda_lib.quantize_mx_fit(dev(b), 0, ws=ws)
        torch.cuda.synchronize()
        o = qn.mxfp4_fit(syn.bf16_bits_to_f32(b))
        np.testing.assert_array_equal(ft.table.cpu().numpy().view(np.uint32), o.table.view(np.uint32))
        np.testing.assert_array_equal(ft.levels.cpu().numpy(), o.q)
        np.testing.assert_array_equal(ft.codes.cpu().numpy(), fm.pack_codes(o.codes))
    one = np.full((16, 64), 0x40F0, dtype=np.uint16)          # 7.5 everywhere: s = 1.25 in every group
    ft = cuda_lib.quantize_mx_fit(dev(one), 0, ws=ws)
    torch.cuda.synchronize()
    assert np.all(ft.table.cpu().numpy() == np.float32(1.25)) and np.all(ft.levels.cpu().numpy() == 255)
    assert cuda_lib.get_last_error() == 0
