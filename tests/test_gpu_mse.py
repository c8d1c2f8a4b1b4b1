"""GPU parity of the NVFP4 MSE-optimal scale search (fp4_quantize_mse)
against the oracle: codes, scale bytes and tensor-scale bits bit-exact after
every number of alternations, including a tensor large enough that the
tensor-scale step sums more than 1024 block partials per thread group."""
import numpy as np
import pytest
import torch

from fp4_microscaled_quantized_b200 import synthetic as syn
from oracle import formats as fm
from oracle import quant as qn

pytestmark = pytest.mark.gpu


def to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def f32_bits(v):
    return np.float32(v).view(np.uint32)


def assert_qt_equal(g, o):
    torch.cuda.synchronize()
    np.testing.assert_array_equal(g.codes.cpu().numpy(), fm.pack_codes(o.codes), err_msg="codes")
    np.testing.assert_array_equal(g.scales.cpu().numpy(), o.scales, err_msg="scales")
    np.testing.assert_array_equal(g.scales_swz.cpu().numpy(), qn.swizzle_scales(o.scales), err_msg="swizzled")
    assert g.tensor_scale.cpu().numpy().view(np.uint32)[0] == f32_bits(o.tensor_scale)


def _input(kind, shape, seed):
    if kind == "gauss":
        return syn.gaussian(shape, 1.0, seed)
    if kind == "t3":
        return syn.student_t(shape, seed, scale=0.02)
    return syn.outlier_elements(shape, seed)


@pytest.mark.parametrize("shape,iters,kind", [
    ((64, 256), 0, "gauss"), ((64, 256), 2, "t3"), ((40, 96), 1, "outlier"),
    ((136, 512), 3, "t3"), ((8, 32), 2, "gauss")])
def test_mse_search_parity(cuda_lib, shape, iters, kind):
    bits = _input(kind, shape, seed=31 + iters)
    x = syn.bf16_bits_to_f32(bits)
    g = cuda_lib.quantize_mse(to_dev(bits), iters)
    o = qn.nvfp4_mse_search(x, iters)
    assert_qt_equal(g, o)
    assert cuda_lib.get_last_error() == 0


def test_mse_search_tiled_large_tensor(cuda_lib):
    """10240 x 4096 elements (5120 blocks of 8192: the tensor-scale step's
    threads each sum runs of 8 partials): the input repeats one 64-row slab,
    so the oracle's group step on the slab (at the tensor's own s_T) gives
    every row, and its tensor-scale step runs on the whole tensor."""
    slab = syn.student_t((64, 4096), seed=41, scale=0.02)
    bits = np.tile(slab, (160, 1))
    xs = syn.bf16_bits_to_f32(slab)
    s_T0 = qn.nvfp4_tensor_scale(qn.abs_max(xs), qn.NV_RTN_DIV)
    xg = xs.reshape(64, -1, 16)

    def group(s_T):
        s8 = qn.mse_group_scales(xg, s_T)
        d = (fm.e4m3_value(s8).astype(np.float32) * np.float32(s_T)).astype(np.float32)
        codes, _, _ = qn._encode_rtn(xg, d)
        return s8, codes

    s8_0, c0 = group(s_T0)
    x_full = syn.bf16_bits_to_f32(bits)
    s_T1 = qn.mse_tensor_scale(x_full, np.tile(s8_0, (160, 1)), np.tile(c0, (160, 1, 1)), s_T0)
    assert s_T1 != s_T0
    s8_1, c1 = group(s_T1)
    g = cuda_lib.quantize_mse(to_dev(bits), 1)
    torch.cuda.synchronize()
    assert g.tensor_scale.cpu().numpy().view(np.uint32)[0] == f32_bits(s_T1)
    np.testing.assert_array_equal(g.scales.cpu().numpy(), np.tile(s8_1, (160, 1)))
    np.testing.assert_array_equal(g.codes.cpu().numpy(), np.tile(fm.pack_codes(c1.reshape(64, -1)), (160, 1)))
    assert cuda_lib.get_last_error() == 0


def test_mse_search_not_worse_than_rtn_or_four_over_six(cuda_lib):
    """At a layer's size (4096 x 4096), from the library's outputs alone:
    every group's error under the searched scale is at most its error under
    RTN and Four-Over-Six (same tensor scale), and one alternation does not
    raise the total error."""
    bits = syn.student_t((4096, 4096), seed=43, scale=0.02)
    x = to_dev(bits)
    xd = x.double()

    def group_err(q):
        return ((cuda_lib.dequantize(q).double() - xd) ** 2).view(4096, -1, 16).sum(-1)

    # slack for the de-quantised values' own rounding (fp32(fp32(q s8) s_T)
    # here, fp32(q fp32(s8 s_T)) in the search's error)
    slack = 1e-9 * (xd ** 2).view(4096, -1, 16).sum(-1)

    m0 = cuda_lib.quantize_mse(x, 0)
    m1 = cuda_lib.quantize_mse(x, 1)
    r = cuda_lib.quantize(x, qn.NVFP4, qn.RTN, 0)
    f = cuda_lib.quantize(x, qn.NVFP4, qn.FOUR_OVER_SIX, 0)
    assert torch.equal(m0.tensor_scale, r.tensor_scale)
    e0, er, ef = group_err(m0), group_err(r), group_err(f)
    assert bool((e0 <= er * (1 + 1e-5) + slack).all()) and bool((e0 <= ef * (1 + 1e-5) + slack).all())
    assert float(e0.sum()) < 0.97 * float(ef.sum())
    assert float(group_err(m1).sum()) <= float(e0.sum()) * (1 + 1e-6)
    assert cuda_lib.get_last_error() == 0


def test_mse_search_arguments_and_launches(cuda_lib):
    x = to_dev(syn.gaussian((64, 256), 1.0, seed=2))
    for cols_x, iters, status in ((to_dev(syn.gaussian((64, 48), 1.0, seed=2)), 0, 1), (x, 65, 1), (x, -1, 1)):
        with pytest.raises(cuda_lib.Fp4Error) as e:
            cuda_lib.quantize_mse(cols_x, iters)
        assert e.value.status == status
    with pytest.raises(cuda_lib.Fp4Error) as e:
        cuda_lib.quantize_mse(x, 0, ws=torch.empty(64, dtype=torch.uint8, device="cuda"))
    assert e.value.status == 4
    assert cuda_lib.quantize_mse_workspace_size(64, 256) == 256 + 256
    empty = cuda_lib.quantize_mse(torch.empty((0, 256), dtype=torch.bfloat16, device="cuda"), 2)
    assert empty.rows == 0
    for iters in (0, 3):
        n0 = cuda_lib.launch_count()
        cuda_lib.quantize_mse(x, iters)
        # amax, (iters + 1) group steps, iters tensor-scale steps, swizzle padding (64 rows)
        assert cuda_lib.launch_count() - n0 == 2 + 2 * iters + 1


def test_mse_search_flags_non_finite_input(cuda_lib):
    bits = syn.gaussian((32, 64), 1.0, seed=3)
    bits[5, 7] = 0x7FC0                                   # bf16 NaN
    cuda_lib.get_last_error()
    cuda_lib.quantize_mse(to_dev(bits), 1)
    assert cuda_lib.get_last_error() == 6
