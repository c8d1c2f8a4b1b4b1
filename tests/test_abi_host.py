"""Host-side logic of the C ABI, on the CPU: every argument check below
returns before the library touches the CUDA runtime (no device memory is
read or written; the device pointers passed are never dereferenced), so
these run without a GPU.  Status codes as include/fp4.h defines them."""
import ctypes
import os

import pytest

from fp4_microscaled_quantized_b200 import api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "fp4_microscaled_quantized_b200", "libfp4_b200.so")

OK, INVALID, UNSUPPORTED, ALIGNMENT, WORKSPACE = 0, 1, 2, 3, 4
FAKE = 0x100000          # a 16-byte aligned address that is never dereferenced


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        from fp4_microscaled_quantized_b200 import build
        build.build()
    lib = ctypes.CDLL(LIB)
    api._declare(lib)
    f = lib.fp4_quantize_mse
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                  ctypes.POINTER(api.fp4_qtensor), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    for name, args in (("fp4_dequantize", [ctypes.POINTER(api.fp4_qtensor), ctypes.c_void_p, ctypes.c_int32,
                                           ctypes.c_void_p]),
                       ("fp4_transpose_square16", [ctypes.POINTER(api.fp4_qtensor),
                                                   ctypes.POINTER(api.fp4_qtensor), ctypes.c_void_p])):
        getattr(lib, name).restype = ctypes.c_int
        getattr(lib, name).argtypes = args
    return lib


def fake_out():
    q = api.fp4_qtensor()
    q.codes, q.scales, q.tensor_scale = FAKE, FAKE + 0x1000, FAKE + 0x2000
    return q


def quantize(lib, x, in_rows, in_cols, fmt, rnd, group, had=0, transpose=0, out=None):
    out = out if out is not None else fake_out()
    return lib.fp4_quantize(x, in_rows, in_cols, transpose, fmt, rnd, group, api.fp4_had(had, 0, 0), 0, 0,
                            ctypes.byref(out), None, 0, None)


@pytest.mark.parametrize("fmt,rnd,group,had,shape,transpose,want", [
    (2, 0, 16, 0, (64, 64), 0, INVALID),                     # unknown format
    (1, 6, 16, 0, (64, 64), 0, INVALID),                     # unknown rounding
    (1, 0, 32, 0, (64, 64), 0, UNSUPPORTED),                 # NVFP4 groups are 16
    (1, 4, 16, 0, (64, 128), 0, UNSUPPORTED),                # MS-EDEN needs a rotation
    (1, 4, 16, 8, (64, 128), 0, UNSUPPORTED),                # block 8: not a rotation size
    (0, 2, 32, 0, (64, 64), 0, UNSUPPORTED),                 # Four-Over-Six is NVFP4-only
    (1, 0, 16, 48, (64, 96), 0, UNSUPPORTED),                # block 48
    (1, 5, 16, 0, (72, 64), 0, INVALID),                     # square blocks: whole 16 x 16 blocks
    (1, 5, 16, 16, (64, 64), 0, UNSUPPORTED),                # square blocks take no rotation
    (1, 0, 16, 0, (64, 24), 0, INVALID),                     # inner dim not a multiple of 16
    (1, 0, 16, 64, (64, 96), 0, INVALID),                    # ... nor of the rotation block
    (1, 0, 16, 0, (64, 36), 1, ALIGNMENT),                   # transposed: input rows of 36 (not 8k) elements
    (1, 0, 16, 0, (40, 64), 1, INVALID),                     # transposed inner dim 40 not a multiple of 16
    (1, 0, 16, 256, (256, 64), 1, WORKSPACE),                # transposed 256-blocks: valid, no workspace given
])
def test_quantize_argument_checks(lib, fmt, rnd, group, had, shape, transpose, want):
    assert quantize(lib, FAKE, shape[0], shape[1], fmt, rnd, group, had, transpose) == want


def test_quantize_pointer_checks_and_empty_tensor(lib):
    out = api.fp4_qtensor()                                    # all pointers null
    assert quantize(lib, FAKE, 0, 64, 1, 0, 16, out=out) == OK
    assert (out.rows, out.cols, out.fmt) == (0, 64, 1)
    assert quantize(lib, FAKE, 32, 64, 1, 0, 16, out=out) == INVALID
    assert lib.fp4_quantize(FAKE, 32, 64, 0, 1, 0, 16, api.fp4_had(0, 0, 0), 0, 0, None, None, 0, None) == INVALID
    assert quantize(lib, None, 32, 64, 1, 0, 16) == INVALID
    assert quantize(lib, FAKE + 8, 32, 64, 1, 0, 16) == ALIGNMENT
    misaligned = fake_out()
    misaligned.codes = FAKE + 4
    assert quantize(lib, FAKE, 32, 64, 1, 0, 16, out=misaligned) == ALIGNMENT


def test_quantize_mse_argument_checks(lib):
    q = lib.fp4_quantize_mse
    out = fake_out()
    assert q(FAKE, 64, 48, 0, ctypes.byref(out), FAKE, 1 << 20, None) == INVALID      # cols % 32
    assert q(FAKE, 64, 256, 65, ctypes.byref(out), FAKE, 1 << 20, None) == INVALID    # iters > 64
    assert q(FAKE, 64, 256, -1, ctypes.byref(out), FAKE, 1 << 20, None) == INVALID
    assert q(FAKE, 64, 256, 0, None, FAKE, 1 << 20, None) == INVALID
    assert q(None, 64, 256, 0, ctypes.byref(out), FAKE, 1 << 20, None) == INVALID
    assert q(FAKE + 2, 64, 256, 0, ctypes.byref(out), FAKE, 1 << 20, None) == ALIGNMENT
    assert q(FAKE, 64, 256, 0, ctypes.byref(out), FAKE, 511, None) == WORKSPACE         # needs 512
    assert q(FAKE, 64, 256, 0, ctypes.byref(out), None, 0, None) == WORKSPACE
    assert q(FAKE, 64, 256, 0, ctypes.byref(out), FAKE + 8, 512, None) == ALIGNMENT
    empty = api.fp4_qtensor()
    assert q(None, 0, 256, 3, ctypes.byref(empty), None, 0, None) == OK
    assert (empty.rows, empty.cols, empty.fmt) == (0, 256, 1)


def test_requantize_dequantize_transpose_checks(lib):
    src = fake_out()
    src.rows, src.cols, src.fmt = 64, 64, 1
    out = fake_out()
    rq = lambda qin, rnd, had=0, tr=1: lib.fp4_requantize(  # noqa: E731
        qin, tr, rnd, api.fp4_had(had, 0, 0), 0, 0, ctypes.byref(out), None, 0, None)
    assert rq(None, 0) == INVALID
    assert rq(ctypes.byref(src), 5) == UNSUPPORTED                          # square blocks: bf16 input only
    assert rq(ctypes.byref(src), 9) == INVALID
    bad = fake_out()
    bad.rows, bad.cols, bad.fmt = 64, 64, 3
    assert rq(ctypes.byref(bad), 0) == INVALID
    assert lib.fp4_dequantize(ctypes.byref(src), FAKE, 2, None) == INVALID   # output dtype
    odd = fake_out()
    odd.rows, odd.cols, odd.fmt = 64, 40, 1
    assert lib.fp4_dequantize(ctypes.byref(odd), FAKE, 0, None) == INVALID   # cols % 16
    none = api.fp4_qtensor()
    none.rows, none.cols, none.fmt = 0, 64, 1
    assert lib.fp4_dequantize(ctypes.byref(none), None, 0, None) == OK
    mx = fake_out()
    mx.rows, mx.cols, mx.fmt = 64, 64, 0
    assert lib.fp4_transpose_square16(ctypes.byref(mx), ctypes.byref(out), None) == INVALID
    small = fake_out()
    small.rows, small.cols, small.fmt = 48, 64, 1
    assert lib.fp4_transpose_square16(ctypes.byref(small), ctypes.byref(out), None) == INVALID


PRESETS = {  # id: (fmt, fwd_rounding, fwd_had, bwd_rounding, bwd_had, randomized, mask, w_rounding, w_reuse)
    0: (0, 1, 32, 3, 32, 1, 1, -1, 0),        # Quartet: MXFP4, H32 + QuEST, RHT32 + SR, mask epilogue
    1: (1, 2, 0, 4, 128, 1, 0, -1, 0),        # Quartet II: NVFP4, 4/6, RHT128 + MS-EDEN
    2: (1, 0, 0, 0, 0, 0, 0, -1, 0),          # NVFP4 RTN
    3: (1, 0, 0, 3, 128, 1, 0, -1, 0),        # simplified TetraJet-v2: RTN fwd, RHT128 + SR bwd
    4: (1, 0, 0, 3, 16, 1, 0, 5, 1),          # NVIDIA: square-block W re-used in the dX GEMM
}


@pytest.mark.parametrize("pid", sorted(PRESETS))
def test_recipe_presets(lib, pid):
    r = api.fp4_recipe()
    assert lib.fp4_recipe_preset(pid, ctypes.byref(r)) == OK
    got = (r.fmt, r.fwd_rounding, r.fwd_had, r.bwd_rounding, r.bwd_had, r.bwd_randomized, r.mask_epilogue,
           r.w_rounding, r.w_reuse)
    assert got == PRESETS[pid]
    assert (r.out_y, r.out_dx, r.out_dw) == (0, 0, 0)
    assert lib.fp4_linear_workspace_size(ctypes.byref(r), 256, 512, 1024, 0) > 0 or pid == 0
    assert lib.fp4_linear_workspace_size(ctypes.byref(r), 256, 512, 1024, 1) > 0


def test_recipe_validation(lib):
    r = api.fp4_recipe()
    assert lib.fp4_recipe_preset(99, ctypes.byref(r)) == INVALID
    assert lib.fp4_recipe_preset(0, None) == INVALID
    lib.fp4_recipe_preset(2, ctypes.byref(r))
    r.w_reuse = 1                                            # re-use needs square-block weights
    assert lib.fp4_linear_workspace_size(ctypes.byref(r), 256, 512, 1024, 1) == 0
    lib.fp4_recipe_preset(1, ctypes.byref(r))
    r.mask_epilogue = 1                                      # the mask epilogue needs QuEST + H32
    assert lib.fp4_linear_workspace_size(ctypes.byref(r), 256, 512, 1024, 1) == 0
    lib.fp4_recipe_preset(1, ctypes.byref(r))
    r.out_dw = 2
    assert lib.fp4_linear_workspace_size(ctypes.byref(r), 256, 512, 1024, 1) == 0
    ctx = api.fp4_ctx()
    assert lib.fp4_linear_fwd(FAKE, FAKE, 256, 512, 1024, ctypes.byref(r), 0, FAKE, ctypes.byref(ctx),
                              FAKE, 1 << 30, None) == INVALID


def _noalloc(lib, x, in_rows, in_cols, fmt, rnd, group, had=0, transpose=0, out=None):
    f = lib.fp4_quantize_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                  ctypes.c_int32, ctypes.c_int32, api.fp4_had, ctypes.c_uint64, ctypes.c_uint32,
                  ctypes.POINTER(api.fp4_qtensor), ctypes.c_void_p]
    out = out if out is not None else fake_out()
    return f(x, in_rows, in_cols, transpose, fmt, rnd, group, api.fp4_had(had, 0, 0), 0, 0, ctypes.byref(out), None)


@pytest.mark.parametrize("fmt,rnd,group,had,shape,transpose,want", [
    # a tensor far larger than the 4 MiB scratch: the argument errors still come first
    (1, 4, 16, 8, (8192, 8192), 0, UNSUPPORTED),            # MS-EDEN with block 8
    (1, 4, 16, 48, (8192, 8160), 0, UNSUPPORTED),           # MS-EDEN with block 48
    (1, 4, 16, 128, (8192, 8200), 0, INVALID),              # inner dim not a multiple of 128
    (1, 0, 32, 0, (8192, 8192), 0, UNSUPPORTED),            # wrong group for NVFP4
    (1, 4, 16, 128, (8192, 8196), 1, ALIGNMENT),            # transposed: input rows of 8196 elements
    # valid arguments beyond the scratch: the size check
    (1, 4, 16, 128, (8192, 8192), 0, WORKSPACE),
    (1, 5, 16, 0, (32768, 16384), 0, WORKSPACE),            # square blocks: 256 + rows * cols / 64 bytes
])
def test_quantize_noalloc_status_matches_quantize(lib, fmt, rnd, group, had, shape, transpose, want):
    """fp4_quantize_noalloc returns fp4_quantize's status for an invalid
    argument, whatever the tensor's size; only valid arguments reach its own
    scratch-size check (all before any CUDA call)."""
    assert _noalloc(lib, FAKE, shape[0], shape[1], fmt, rnd, group, had, transpose) == want
    if want != WORKSPACE:
        assert quantize(lib, FAKE, shape[0], shape[1], fmt, rnd, group, had, transpose) == want


def test_quantize_noalloc_square_block_limit(lib):
    """The square-block mode keeps one fp32 maximum per 16 x 16 block in the
    scratch: 256 + rows * cols / 64 bytes, so 4 MiB holds about 268 million
    elements."""
    need = lib.fp4_quantize_workspace_size(16384, 16352, 1, 5, 0)
    assert need == 256 + 16384 * 16352 // 64
    assert need <= 4 << 20
    assert lib.fp4_quantize_workspace_size(16384, 16384, 1, 5, 0) > 4 << 20
    empty = api.fp4_qtensor()
    assert _noalloc(lib, None, 0, 64, 1, 5, 16, out=empty) == OK


def test_transform_and_fit_argument_checks(lib):
    """fp4_block_transform, fp4_quantize_f32 and fp4_quantize_mx_fit return
    their argument errors before any CUDA call."""
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    bt = lib.fp4_block_transform
    bt.restype, bt.argtypes = ctypes.c_int, [P, P, I64, I64, I32, I32, P, SZ, P]
    lib.fp4_block_transform_workspace_size.restype = SZ
    lib.fp4_block_transform_workspace_size.argtypes = [I32]
    assert lib.fp4_block_transform_workspace_size(256) == 256 * 256 * 4
    assert lib.fp4_block_transform_workspace_size(48) == 0
    assert bt(FAKE, FAKE, 8, 64, 3, 16, FAKE, 1 << 20, None) == UNSUPPORTED      # kind (GSR has no value)
    assert bt(FAKE, FAKE, 8, 64, 1, 48, FAKE, 1 << 20, None) == UNSUPPORTED      # block
    assert bt(FAKE, FAKE, 8, 80, 1, 32, FAKE, 1 << 20, None) == INVALID          # cols % block
    assert bt(FAKE + 4, FAKE, 8, 64, 1, 16, FAKE, 1 << 20, None) == ALIGNMENT
    assert bt(FAKE, FAKE, 8, 64, 2, 16, FAKE, 1023, None) == WORKSPACE           # needs 1024
    assert bt(None, None, 0, 64, 1, 16, None, 0, None) == OK                      # empty
    qf = lib.fp4_quantize_f32
    qf.restype = ctypes.c_int
    qf.argtypes = [P, I64, I64, I32, I32, I32, ctypes.c_uint64, ctypes.c_uint32,
                   ctypes.POINTER(api.fp4_qtensor), P, SZ, P]
    out = fake_out()
    assert qf(FAKE, 8, 64, 1, 4, 16, 0, 0, ctypes.byref(out), FAKE, 1 << 20, None) == UNSUPPORTED   # MS-EDEN
    assert qf(FAKE, 8, 64, 1, 5, 16, 0, 0, ctypes.byref(out), FAKE, 1 << 20, None) == UNSUPPORTED   # square
    assert qf(FAKE, 8, 64, 0, 2, 32, 0, 0, ctypes.byref(out), FAKE, 1 << 20, None) == UNSUPPORTED   # MX 4/6
    assert qf(FAKE, 8, 48, 1, 0, 16, 0, 0, ctypes.byref(out), FAKE, 1 << 20, None) == INVALID       # cols % 32
    assert qf(FAKE + 8, 8, 64, 1, 0, 16, 0, 0, ctypes.byref(out), FAKE, 1 << 20, None) == ALIGNMENT
    assert qf(FAKE, 8, 64, 1, 0, 16, 0, 0, ctypes.byref(out), None, 0, None) == WORKSPACE
    mf = lib.fp4_quantize_mx_fit
    mf.restype, mf.argtypes = ctypes.c_int, [P, I64, I64, I32, P, P, P, P, SZ, P]
    lib.fp4_quantize_mx_fit_workspace_size.restype = SZ
    assert lib.fp4_quantize_mx_fit_workspace_size() >= 256 + 255 * 4
    assert mf(FAKE, 8, 64, 48, FAKE, FAKE, FAKE, FAKE, 4096, None) == UNSUPPORTED      # had block
    assert mf(FAKE, 8, 48, 0, FAKE, FAKE, FAKE, FAKE, 4096, None) == INVALID            # cols % 32
    assert mf(FAKE, 8, 64, 128, FAKE, FAKE, FAKE, FAKE, 4096, None) == INVALID          # cols % had
    assert mf(FAKE, 8, 64, 0, FAKE, FAKE, FAKE, FAKE, 100, None) == WORKSPACE
    assert mf(FAKE, 8, 64, 0, None, FAKE, FAKE, FAKE, 4096, None) == INVALID
    assert mf(FAKE + 2, 8, 64, 0, FAKE, FAKE, FAKE, FAKE, 4096, None) == ALIGNMENT


def test_binding_rejects_outputs_of_the_wrong_shape():
    """The C ABI sees only an output's pointer, so the binding checks a
    caller-given output's shape before the call (no device work here)."""
    import torch
    from fp4_microscaled_quantized_b200 import api

    class Fake:
        rows, cols = 4, 64
        codes = torch.empty((4, 32), dtype=torch.uint8)

    with pytest.raises(AssertionError):
        api.gemm(Fake(), Fake(), out=torch.empty((4, 5)))
    with pytest.raises(AssertionError):
        api.dequantize(Fake(), out=torch.empty((4, 32)))
    with pytest.raises(AssertionError):
        api.dequantize(Fake(), out=torch.empty((64, 4)).t())          # right shape, not contiguous
