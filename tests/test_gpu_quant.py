"""GPU parity of the Hadamard / quantise / pack / swizzle kernels against the
oracle: bit-exact codes, scale bytes, tensor-scale bits and mask bits in
every mode (the stochastic ones draw the same Philox bits)."""
import numpy as np
import pytest
import torch

from fp4_microscaled_quantized_b200 import synthetic as syn
from oracle import formats as fm
from oracle import hadamard as hd
from oracle import quant as qn

pytestmark = pytest.mark.gpu

COMBOS = [(f, r, h) for f in (qn.MXFP4, qn.NVFP4) for r in range(5) for h in (0, 16, 32, 64, 128, 256)
          if qn.supported(f, r, h)]


def to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def assert_qt_equal(g, o, check_mask=True):
    torch.cuda.synchronize()
    np.testing.assert_array_equal(g.codes.cpu().numpy(), fm.pack_codes(o.codes), err_msg="codes")
    np.testing.assert_array_equal(g.scales.cpu().numpy(), o.scales, err_msg="scales")
    swz = g.scales_swz.cpu().numpy()
    np.testing.assert_array_equal(swz, qn.swizzle_scales(o.scales), err_msg="swizzled scales")
    assert g.tensor_scale.cpu().numpy().view(np.uint32)[0] == np.float32(o.tensor_scale).view(np.uint32)
    if check_mask and o.mask is not None:
        np.testing.assert_array_equal(g.mask.cpu().numpy(), fm.pack_mask(o.mask), err_msg="mask")


@pytest.mark.parametrize("fmt,rnd,had", COMBOS)
@pytest.mark.parametrize("transpose", [False, True])
def test_quantize_parity(cuda_lib, fmt, rnd, had, transpose):
    shape = (512, 200) if transpose else (200, 512)
    bits = syn.outlier_elements(shape, seed=7, stream=fmt * 10 + rnd)
    x = syn.bf16_bits_to_f32(bits)
    seed, stag, ttag = 0x1234ABCD5678, 1, 9
    g = cuda_lib.quantize(to_dev(bits), fmt, rnd, had, randomized=had > 0, seed=seed,
                          sign_tag=stag, tensor_tag=ttag, transpose=transpose)
    o = qn.quantize(x, fmt, rnd, had, had > 0, seed, stag, ttag, transpose=transpose)
    assert_qt_equal(g, o)
    assert cuda_lib.get_last_error() == 0


@pytest.mark.parametrize("fmt,fwd_rnd,rnd,had", [
    (qn.NVFP4, qn.FOUR_OVER_SIX, qn.MS_EDEN, 128), (qn.NVFP4, qn.FOUR_OVER_SIX, qn.SR, 16),
    (qn.NVFP4, qn.FOUR_OVER_SIX, qn.MS_EDEN, 64),
    (qn.NVFP4, qn.RTN, qn.RTN, 0), (qn.MXFP4, qn.QUEST, qn.SR, 32), (qn.MXFP4, qn.RTN, qn.QUEST, 32)])
@pytest.mark.parametrize("transpose", [True, False])
def test_requantize_parity(cuda_lib, fmt, fwd_rnd, rnd, had, transpose):
    """De-quantise a saved (oracle-quantised) tensor, transpose, rotate,
    quantise again (Quartet II computation graph, backward steps 1-4)."""
    bits = syn.student_t((384, 256), seed=3, unit_rms=True)
    x = syn.bf16_bits_to_f32(bits)
    saved = qn.quantize(x, fmt, fwd_rnd, 0)
    dev = cuda_lib.alloc_qtensor(384, 256, fmt, mask=False)
    dev.codes.copy_(torch.from_numpy(fm.pack_codes(saved.codes)))
    dev.scales.copy_(torch.from_numpy(saved.scales))
    dev.tensor_scale.copy_(torch.tensor([float(saved.tensor_scale)], dtype=torch.float32))
    seed = 77
    g = cuda_lib.requantize(dev, rnd, had, randomized=had > 0, seed=seed, sign_tag=2, tensor_tag=4,
                            transpose=transpose)
    o = qn.requantize(saved, rnd, had, had > 0, seed, 2, 4, transpose=transpose)
    assert_qt_equal(g, o)


@pytest.mark.parametrize("fmt,fwd_rnd,rnd", [(qn.NVFP4, qn.FOUR_OVER_SIX, qn.MS_EDEN), (qn.NVFP4, qn.RTN, qn.SR),
                                          (qn.MXFP4, qn.QUEST, qn.SR)])
def test_requantize_transposed_256_blocks(cuda_lib, fmt, fwd_rnd, rnd):
    """Re-quantisation of a saved tensor, transposed, with 256-element
    rotation blocks (the transposed kernel's 256-row tile); 176 input
    columns (NVFP4) leave a ragged last 32-column tile, MXFP4 groups need
    224."""
    cols = 176 if fmt == qn.NVFP4 else 224
    bits = syn.student_t((512, cols), seed=4, unit_rms=True)
    saved = qn.quantize(syn.bf16_bits_to_f32(bits), fmt, fwd_rnd, 0)
    dev = cuda_lib.alloc_qtensor(512, cols, fmt, mask=False)
    dev.codes.copy_(torch.from_numpy(fm.pack_codes(saved.codes)))
    dev.scales.copy_(torch.from_numpy(saved.scales))
    dev.tensor_scale.copy_(torch.tensor([float(saved.tensor_scale)], dtype=torch.float32))
    g = cuda_lib.requantize(dev, rnd, 256, randomized=True, seed=91, sign_tag=1, tensor_tag=2, transpose=True)
    o = qn.requantize(saved, rnd, 256, True, 91, 1, 2, transpose=True)
    assert_qt_equal(g, o)
    assert cuda_lib.get_last_error() == 0


@pytest.mark.parametrize("block", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("randomized", [False, True])
def test_hadamard_parity(cuda_lib, block, randomized):
    bits = syn.gaussian((96, 512), 1.0, seed=5)
    y = cuda_lib.hadamard(to_dev(bits), block, randomized, seed=42, sign_tag=3)
    o = hd.block_transform(syn.bf16_bits_to_f32(bits), block, randomized, 42, 3)
    np.testing.assert_array_equal(y.cpu().numpy().view(np.uint32), o.view(np.uint32))


def test_swizzle_kernel(cuda_lib):
    s = np.random.default_rng(0).integers(0, 255, (300, 10)).astype(np.uint8)
    out = cuda_lib.swizzle_scales(torch.from_numpy(s).cuda())
    np.testing.assert_array_equal(out.cpu().numpy(), qn.swizzle_scales(s))


def test_multi_tile_large_parity(cuda_lib):
    """Several row tiles, a ragged row count and a 4096-wide inner dimension
    through the grid-stride loop (config-5 row length)."""
    bits = syn.quantizer_sweep(4096 * 1000 + 4096 * 37, seed=7)
    x = syn.bf16_bits_to_f32(bits)
    for fmt, rnd, had in [(qn.NVFP4, qn.MS_EDEN, 128), (qn.NVFP4, qn.FOUR_OVER_SIX, 0),
                          (qn.MXFP4, qn.SR, 32)]:
        g = cuda_lib.quantize(to_dev(bits), fmt, rnd, had, randomized=True, seed=5, sign_tag=0,
                              tensor_tag=1)
        o = qn.quantize(x, fmt, rnd, had, True, 5, 0, 1)
        assert_qt_equal(g, o)


def test_nonfinite_input_flags_status(cuda_lib):
    bits = syn.gaussian((64, 256), 1.0, seed=1)
    bits[3, 17] = 0x7FC0                                   # NaN
    for fmt, rnd, had in [(qn.NVFP4, qn.RTN, 0), (qn.NVFP4, qn.MS_EDEN, 128), (qn.MXFP4, qn.QUEST, 32)]:
        cuda_lib.quantize(to_dev(bits), fmt, rnd, had, randomized=True)
        assert cuda_lib.get_last_error() == 6
        assert cuda_lib.get_last_error() == 0              # cleared by the read


def test_argument_errors(cuda_lib):
    x = to_dev(syn.gaussian((64, 256), 1.0, seed=1))
    with pytest.raises(cuda_lib.Fp4Error) as e:
        cuda_lib.quantize(x, qn.MXFP4, qn.MS_EDEN, 128)
    assert e.value.status == 2
    with pytest.raises(cuda_lib.Fp4Error) as e:
        cuda_lib.quantize(x, qn.NVFP4, qn.MS_EDEN, 0)
    assert e.value.status == 2
    with pytest.raises(cuda_lib.Fp4Error) as e:
        cuda_lib.quantize(to_dev(syn.gaussian((64, 200), 1.0, 1)), qn.NVFP4, qn.RTN, 128)
    assert e.value.status == 1                             # 200 % 128 != 0
    with pytest.raises(cuda_lib.Fp4Error) as e:
        cuda_lib.quantize(x, qn.NVFP4, qn.MS_EDEN, 128, ws=cuda_lib.alloc_workspace(16))
    assert e.value.status == 4


def test_empty_input_is_a_noop(cuda_lib):
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    q = cuda_lib.quantize(x, qn.NVFP4, qn.MS_EDEN, 128)
    assert q.rows == 0 and cuda_lib.get_last_error() == 0


def test_hardware_e2m1_encoder_exhaustive(cuda_lib):
    """The hardware conversion used by the 32-per-lane path equals the
    per-element round-to-nearest-even onto E2M1 for every fp32 input, and the
    hardware decoder gives the code table's value for every code pair."""
    assert cuda_lib.selftest_e2m1() == 0


def test_exact_scale_arithmetic(cuda_lib):
    """The corrected divisions and the E8M3 reciprocal of the NVFP4 scale
    path equal CUDA's correctly rounded __fdiv_rn / __frcp_rn on every case
    checked, and the hardware E4M3 conversions equal the scale rounding and
    the code table."""
    assert cuda_lib.selftest_arith() == [0, 0, 0, 0, 0, 0]


@pytest.mark.parametrize("fmt,rnd,had", [(qn.NVFP4, qn.FOUR_OVER_SIX, 0), (qn.NVFP4, qn.MS_EDEN, 16),
                                         (qn.NVFP4, qn.SR, 16), (qn.NVFP4, qn.QUEST, 0)])
@pytest.mark.parametrize("transpose", [False, True])
def test_narrow_inner_dim_path(cuda_lib, fmt, rnd, had, transpose):
    """Inner dimension 16 mod 32 runs the 8-per-lane kernels."""
    shape = (48, 136) if transpose else (136, 48)
    bits = syn.outlier_elements(shape, seed=9, stream=rnd)
    g = cuda_lib.quantize(to_dev(bits), fmt, rnd, had, randomized=had > 0, seed=3, sign_tag=1,
                          tensor_tag=2, transpose=transpose)
    o = qn.quantize(syn.bf16_bits_to_f32(bits), fmt, rnd, had, had > 0, 3, 1, 2, transpose=transpose)
    assert_qt_equal(g, o)


def test_launch_counter_counts_kernels(cuda_lib):
    x = to_dev(syn.gaussian((128, 256), 1.0, seed=1))        # no swizzle padding to zero
    n0 = cuda_lib.launch_count()
    cuda_lib.quantize(x, qn.NVFP4, qn.MS_EDEN, 128, randomized=True)      # pass 1 + pass 2
    cuda_lib.quantize(x, qn.NVFP4, qn.FOUR_OVER_SIX, 0)                     # amax + quantise
    assert cuda_lib.launch_count() - n0 == 4


@pytest.mark.parametrize("had,transpose", [(0, False), (0, True), (16, False), (128, True)])
def test_four_over_six_grid_ties(cuda_lib, had, transpose):
    """Four-Over-Six on a coarse value grid, where many groups' two candidate
    errors tie exactly or within an ulp: a single product, difference or sum
    of the squared-error evaluation rounded differently flips a pick."""
    bits = syn.grid_values((512, 2048), seed=11, stream=had)
    x = syn.bf16_bits_to_f32(bits)
    g = cuda_lib.quantize(to_dev(bits), qn.NVFP4, qn.FOUR_OVER_SIX, had, transpose=transpose)
    o = qn.quantize(x, qn.NVFP4, qn.FOUR_OVER_SIX, had, transpose=transpose)
    assert_qt_equal(g, o)


@pytest.mark.parametrize("had,transpose", [(128, False), (128, True), (16, False), (32, True), (64, True),
                                          (256, False)])
def test_ms_eden_first_pass_bit_exact(cuda_lib, had, transpose):
    """MS-EDEN's first-pass results in the workspace -- the bf16 pseudo-scales
    and the EDEN factors S = <y,y> / <y,q p> -- equal the oracle's bit for bit.
    S is a ratio of two fp32 pairwise sums, so this pins every product and
    the order of every sum, which the final scales (a stochastic rounding of
    S p) would show only rarely."""
    shape = (384, 1024)
    bits = syn.student_t(shape, seed=5, stream=had, unit_rms=True)
    x = syn.bf16_bits_to_f32(bits)
    rows, cols = (shape[1], shape[0]) if transpose else shape
    ws = cuda_lib.alloc_workspace(cuda_lib.workspace_size(rows, cols, qn.NVFP4, qn.MS_EDEN, had))
    seed = 0xC0FFEE
    g = cuda_lib.quantize(to_dev(bits), qn.NVFP4, qn.MS_EDEN, had, randomized=True, seed=seed, sign_tag=1,
                          tensor_tag=2, transpose=transpose, ws=ws)
    o = qn.quantize(x, qn.NVFP4, qn.MS_EDEN, had, True, seed, 1, 2, transpose=transpose)
    torch.cuda.synchronize()
    wsb = ws.cpu().numpy()
    n_pseudo = rows * (cols // 16) * 2
    pseudo = wsb[256:256 + n_pseudo].view(np.uint16).reshape(rows, cols // 16)
    s_off = 256 + (n_pseudo + 255) // 256 * 256
    S = wsb[s_off:s_off + rows * (cols // had) * 4].view(np.uint32).reshape(rows, cols // had)
    np.testing.assert_array_equal(pseudo, (o.extra["pseudo"].view(np.uint32) >> 16).astype(np.uint16))
    np.testing.assert_array_equal(S, o.extra["S"].view(np.uint32))
    assert_qt_equal(g, o)


def test_transposed_block_256_needs_whole_blocks(cuda_lib):
    """Transposed 256-element rotation blocks run on the 256-row tile; the
    quantised tensor's rows (the input's columns) run along the input's 384
    rows, which do not hold whole 256-blocks."""
    x = to_dev(syn.gaussian((384, 256), 1.0, seed=1))      # 384 input rows: not a multiple of 256
    with pytest.raises(cuda_lib.Fp4Error) as e:
        cuda_lib.quantize(x, qn.NVFP4, qn.RTN, 256, transpose=True)
    assert e.value.status == 1                      # FP4_ERR_INVALID_ARG


@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("shape", [(64, 512), (320, 1024), (1024, 96)])
def test_square_block_parity(cuda_lib, shape, transpose):
    """NVFP4 RTN with 16 x 16 block scales: codes, scales (repeated on each
    block's rows) and tensor scale bit-exact against the oracle."""
    in_shape = (shape[1], shape[0]) if transpose else shape
    if (in_shape[0] if transpose else in_shape[1]) % 32:
        pytest.skip("square blocks need 32-element output rows")
    bits = syn.outlier_elements(in_shape, seed=13, stream=shape[0])
    x = syn.bf16_bits_to_f32(bits)
    g = cuda_lib.quantize(to_dev(bits), qn.NVFP4, qn.RTN_SQUARE16, 0, transpose=transpose)
    o = qn.quantize(x, qn.NVFP4, qn.RTN_SQUARE16, 0, transpose=transpose)
    assert_qt_equal(g, o)
    assert cuda_lib.get_last_error() == 0


def test_square_block_transpose_is_the_transpose(cuda_lib):
    """Quantising W^T with 16 x 16 blocks gives the transpose of Q(W) -- the
    property that lets the NVIDIA recipe re-use the forward Q(W) for W^T."""
    bits = syn.gaussian((256, 512), 0.02, seed=4)
    d = to_dev(bits)
    a = cuda_lib.quantize(d, qn.NVFP4, qn.RTN_SQUARE16, 0)
    b = cuda_lib.quantize(d, qn.NVFP4, qn.RTN_SQUARE16, 0, transpose=True)
    torch.cuda.synchronize()
    ca = fm.unpack_codes(a.codes.cpu().numpy())
    cb = fm.unpack_codes(b.codes.cpu().numpy())
    np.testing.assert_array_equal(cb, ca.T)
    sa, sbt = a.scales.cpu().numpy(), b.scales.cpu().numpy()
    np.testing.assert_array_equal(sbt, np.repeat(sa[::16].T, 16, axis=0))


def test_square_block_argument_errors(cuda_lib):
    x = to_dev(syn.gaussian((72, 256), 1.0, seed=1))          # 72 rows: not whole blocks
    with pytest.raises(cuda_lib.Fp4Error) as e:
        cuda_lib.quantize(x, qn.NVFP4, qn.RTN_SQUARE16, 0)
    assert e.value.status == 1
    y = to_dev(syn.gaussian((64, 256), 1.0, seed=1))
    for fmt, had in ((qn.MXFP4, 0), (qn.NVFP4, 16)):
        with pytest.raises(cuda_lib.Fp4Error) as e:
            cuda_lib.quantize(y, fmt, qn.RTN_SQUARE16, had)
        assert e.value.status == 2


@pytest.mark.parametrize("shape", [(64, 128), (256, 512), (640, 192)])
def test_transpose_square16(cuda_lib, shape):
    """fp4_transpose_square16 against the oracle's transpose of the same
    square-block quantised tensor (codes, linear and tensor-core scales,
    tensor scale), and equal to quantising the transposed input directly."""
    bits = syn.outlier_elements(shape, seed=17, stream=shape[1])
    x = syn.bf16_bits_to_f32(bits)
    q = cuda_lib.quantize(to_dev(bits), qn.NVFP4, qn.RTN_SQUARE16, 0)
    t = cuda_lib.transpose_square16(q)
    o = qn.transpose_square16(qn.quantize(x, qn.NVFP4, qn.RTN_SQUARE16, 0))
    assert_qt_equal(t, o)
    d = cuda_lib.quantize(to_dev(bits), qn.NVFP4, qn.RTN_SQUARE16, 0, transpose=True)
    torch.cuda.synchronize()
    assert torch.equal(t.codes, d.codes) and torch.equal(t.scales, d.scales)
