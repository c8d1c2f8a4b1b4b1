"""GPU parity of the tcgen05 block-scaled FP4 GEMM against the fp64 oracle:
|y - y_ref| <= 2^-10 sum_k |a_k b_k| per element (bf16 output adds 2^-9 |y|).
Operands are quantised by the oracle and uploaded, so the GEMM is tested on
its own (scale layout, nibble order, tails, epilogue)."""
import numpy as np
import pytest
import torch

from fp4_microscaled_quantized_b200 import synthetic as syn
from oracle import formats as fm
from oracle import gemm as gm
from oracle import hadamard as hd
from oracle import quant as qn

pytestmark = pytest.mark.gpu


def upload(api, o):
    rows, cols = o.codes.shape
    d = api.alloc_qtensor(rows, cols, o.fmt, mask=o.mask is not None)
    d.codes.copy_(torch.from_numpy(fm.pack_codes(o.codes)))
    d.scales.copy_(torch.from_numpy(o.scales))
    d.scales_swz.copy_(torch.from_numpy(qn.swizzle_scales(o.scales)))
    d.tensor_scale.copy_(torch.tensor([float(o.tensor_scale)], dtype=torch.float32))
    if o.mask is not None:
        d.mask.copy_(torch.from_numpy(fm.pack_mask(o.mask)))
    return d


def operands(fmt, M, N, K, seed):
    rng = np.random.default_rng(seed)
    a = (rng.standard_t(4, (M, K)) * np.exp(rng.uniform(-2, 2, (M, 1)))).astype(np.float32)
    b = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    if fmt == qn.NVFP4:
        return qn.nvfp4_four_over_six(a), qn.nvfp4_rtn(b)
    return qn.mxfp4_quest(hd.block_transform(a, 32, False)), qn.mxfp4_sr(b, 3, 1)


def check(y, y_ref, bound, rel_bf16=False):
    y = y.float().cpu().numpy().astype(np.float64)
    tol = bound + (2.0 ** -9 * np.abs(y_ref) if rel_bf16 else 0)
    err = np.abs(y - y_ref)
    bad = err > tol
    assert not bad.any(), "max excess %g at %s" % ((err - tol).max(), np.argwhere(bad)[:5])


@pytest.mark.parametrize("fmt", [qn.NVFP4, qn.MXFP4])
@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (200, 384, 512), (256, 264, 320), (64, 8, 64),
                                   (1024, 1024, 1024),
                                   # CTA-pair kernel (M > 128): second CTA's rows past M, B tile
                                   # half past N, long K wrapping the 5-stage ring
                                   (300, 136, 192), (384, 640, 1024), (512, 512, 4096), (136, 520, 64)])
def test_gemm_parity(cuda_lib, fmt, M, N, K):
    A, B = operands(fmt, M, N, K, seed=M + N + K)
    y = cuda_lib.gemm(upload(cuda_lib, A), upload(cuda_lib, B))
    y_ref, bound = gm.gemm_ref(A, B)
    check(y, y_ref, bound)


@pytest.mark.parametrize("fmt", [qn.NVFP4, qn.MXFP4])
@pytest.mark.parametrize("M,N,K", [(300, 136, 192), (1024, 1024, 1024)])
def test_gemm_one_cta_kernel(cuda_lib, monkeypatch, fmt, M, N, K):
    """FP4_GEMM_PAIR=0 runs the one-CTA kernel on shapes that otherwise take
    the CTA-pair kernel; both meet the bound."""
    monkeypatch.setenv("FP4_GEMM_PAIR", "0")
    A, B = operands(fmt, M, N, K, seed=M + N + K + 1)
    y = cuda_lib.gemm(upload(cuda_lib, A), upload(cuda_lib, B))
    y_ref, bound = gm.gemm_ref(A, B)
    check(y, y_ref, bound)


@pytest.mark.parametrize("fmt", [qn.NVFP4, qn.MXFP4])
def test_gemm_lossless_exact(cuda_lib, fmt):
    """Grid values with power-of-two scales: every product and partial sum is
    exact in fp32, so the tensor-core result equals the exact product --
    any layout, nibble-order or scale-id mistake shows up as a mismatch."""
    rng = np.random.default_rng(1)
    M, N, K = 256, 256, 512
    g = qn.GROUP[fmt]
    ca = rng.integers(0, 16, (M, K)).astype(np.uint8); ca[:, ::g] = 7
    cb = rng.integers(0, 16, (N, K)).astype(np.uint8); cb[:, ::g] = 7
    # exponent ranges keep every partial sum below 2^20 units of the smallest
    # product, so fp32 accumulation in any order is exact
    lo, hi = (0, 2) if fmt == qn.NVFP4 else (-1, 1)
    ea = rng.integers(lo, hi, (M, K // g)).repeat(g, -1)
    eb = rng.integers(lo, hi, (N, K // g)).repeat(g, -1)
    a = fm.decode_e2m1(ca).astype(np.float64) * np.ldexp(1.0, ea)
    b = fm.decode_e2m1(cb).astype(np.float64) * np.ldexp(1.0, eb)
    A = qn.mxfp4_rtn(a.astype(np.float32)) if fmt == qn.MXFP4 else qn.nvfp4_rtn(a.astype(np.float32))
    B = qn.mxfp4_rtn(b.astype(np.float32)) if fmt == qn.MXFP4 else qn.nvfp4_rtn(b.astype(np.float32))
    y = cuda_lib.gemm(upload(cuda_lib, A), upload(cuda_lib, B)).cpu().numpy().astype(np.float64)
    y_ref, _ = gm.gemm_ref(A, B)
    if fmt == qn.MXFP4:
        np.testing.assert_array_equal(y, a @ b.T)
    np.testing.assert_array_equal(y, y_ref.astype(np.float32).astype(np.float64))


def test_gemm_bf16_output(cuda_lib):
    A, B = operands(qn.NVFP4, 256, 512, 512, seed=9)
    y = cuda_lib.gemm(upload(cuda_lib, A), upload(cuda_lib, B), out_dtype=torch.bfloat16)
    y_ref, bound = gm.gemm_ref(A, B)
    check(y, y_ref, bound, rel_bf16=True)


def test_quartet_epilogue(cuda_lib):
    """dx = 16/9 H32^-1(dx_q (.) (1 - M)) fused into the GEMM epilogue."""
    M, N, K = 256, 512, 256
    rng = np.random.default_rng(4)
    A = qn.mxfp4_sr(rng.standard_normal((M, K)).astype(np.float32), 1, 1)
    B = qn.mxfp4_sr(rng.standard_normal((N, K)).astype(np.float32) * 0.1, 1, 2)
    fwd = qn.mxfp4_quest(hd.block_transform(syn.bf16_bits_to_f32(syn.outlier_channels((M, N), 2)), 32, False))
    mask_dev = torch.from_numpy(fm.pack_mask(fwd.mask)).cuda()
    y = cuda_lib.gemm(upload(cuda_lib, A), upload(cuda_lib, B), mask=mask_dev, inverse_had=32)
    y_ref, bound = gm.gemm_ref(A, B)
    ref, rbound = gm.quartet_epilogue_ref(y_ref, bound, ~fwd.mask)
    check(y, ref, rbound * 1.001 + 1e-30)
    y2 = cuda_lib.gemm(upload(cuda_lib, A), upload(cuda_lib, B), inverse_had=32)
    ref2, rb2 = gm.quartet_epilogue_ref(y_ref, bound, np.ones((M, N), bool))
    check(y2, ref2, rb2 * 1.001 + 1e-30)


def test_gemm_argument_errors(cuda_lib):
    A, B = operands(qn.NVFP4, 128, 256, 256, seed=1)
    dA, dB = upload(cuda_lib, A), upload(cuda_lib, B)
    Am, _ = operands(qn.MXFP4, 128, 256, 256, seed=1)
    with pytest.raises(cuda_lib.Fp4Error) as e:
        cuda_lib.gemm(upload(cuda_lib, Am), dB)
    assert e.value.status == 1
    with pytest.raises(cuda_lib.Fp4Error) as e:
        cuda_lib.gemm(dA, dB, mask=torch.zeros(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == 2
    assert cuda_lib.get_last_error() == 0
