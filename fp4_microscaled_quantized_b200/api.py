"""Python binding of the C-ABI library ``libfp4_b200.so`` (include/fp4.h).

Argument marshalling only: torch provides device memory and the current
stream, every computation runs in the library's CUDA kernels.  There is no
CPU fallback -- without the built library or a CUDA device every call raises.
"""
import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfp4_b200.so")

MXFP4, NVFP4 = 0, 1
RTN, QUEST, FOUR_OVER_SIX, SR, MS_EDEN, RTN_SQUARE16 = 0, 1, 2, 3, 4, 5
GROUP = {MXFP4: 32, NVFP4: 16}

STATUS = {0: "FP4_OK", 1: "FP4_ERR_INVALID_ARG", 2: "FP4_ERR_UNSUPPORTED", 3: "FP4_ERR_ALIGNMENT",
          4: "FP4_ERR_WORKSPACE", 5: "FP4_ERR_CUDA", 6: "FP4_ERR_NONFINITE_INPUT",
          7: "FP4_ERR_TIMEOUT"}


class Fp4Error(RuntimeError):
    def __init__(self, status, what):
        super().__init__("%s failed: %s (%d)" % (what, STATUS.get(status, "?"), status))
        self.status = status


class fp4_had(ctypes.Structure):
    _fields_ = [("block", ctypes.c_int32), ("randomized", ctypes.c_int32),
                ("sign_tag", ctypes.c_uint32)]


class fp4_qtensor(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("scales_swz", ctypes.c_void_p), ("tensor_scale", ctypes.c_void_p),
                ("mask", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("fmt", ctypes.c_int32), ("reserved", ctypes.c_int32)]


_lib = None


def load():
    """Load the library (raises if it is missing or no CUDA device exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libfp4_b200.so is not built (run __graft_entry__.build())")
    lib = ctypes.CDLL(LIB_PATH)
    _declare(lib)
    _lib = lib
    return lib


def _declare(lib):
    P, I32, I64, U32, U64, SZ = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32,
                                 ctypes.c_uint64, ctypes.c_size_t)
    QP = ctypes.POINTER(fp4_qtensor)
    sigs = {
        "fp4_quantize_workspace_size": (SZ, [I64, I64, I32, I32, I32]),
        "fp4_swizzled_scale_bytes": (SZ, [I64, I64]),
        "fp4_hadamard": (ctypes.c_int, [P, P, I64, I64, fp4_had, U64, P]),
        "fp4_quantize": (ctypes.c_int, [P, I64, I64, I32, I32, I32, I32, fp4_had, U64, U32, QP, P, SZ, P]),
        "fp4_requantize": (ctypes.c_int, [QP, I32, I32, fp4_had, U64, U32, QP, P, SZ, P]),
        "fp4_swizzle_scales": (ctypes.c_int, [P, I64, I64, P, P]),
        "fp4_get_last_error": (ctypes.c_int, [P]),
        "fp4_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    }
    for name, (res, args) in sigs.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _declare_extra(lib)


def _declare_extra(lib):
    """Entry points added by later layers (GEMM, linear)."""
    P, I32, I64, U64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t
    QP = ctypes.POINTER(fp4_qtensor)
    RP = ctypes.POINTER(fp4_recipe)
    CP = ctypes.POINTER(fp4_ctx)
    extra = {
        "fp4_gemm": (ctypes.c_int, [QP, QP, P, I32, P, I32, P]),
        "fp4_recipe_preset": (ctypes.c_int, [I32, RP]),
        "fp4_linear_workspace_size": (SZ, [RP, I64, I64, I64, I32]),
        "fp4_linear_fwd": (ctypes.c_int, [P, P, I64, I64, I64, RP, U64, P, CP, P, SZ, P]),
        "fp4_linear_bwd": (ctypes.c_int, [P, CP, I64, I64, I64, RP, U64, P, P, P, SZ, P]),
    }
    for name, (res, args) in extra.items():
        if hasattr(lib, name):
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _check(st, what):
    if st != 0:
        raise Fp4Error(st, what)


def _check_out(t, shape, what):
    """A caller-given output must be a contiguous tensor of the shape the C
    call writes (the C ABI sees only its pointer)."""
    assert tuple(t.shape) == tuple(shape) and t.is_contiguous(), "%s: expected a contiguous %s tensor, got %s" % (
        what, tuple(shape), tuple(t.shape))


@dataclass
class QTensor:
    """A quantised tensor in device memory (rows x cols, groups along cols)."""
    codes: torch.Tensor                    # uint8 rows x cols/2
    scales: Optional[torch.Tensor]         # uint8 rows x cols/g
    scales_swz: Optional[torch.Tensor]     # uint8 tensor-core layout
    tensor_scale: torch.Tensor             # float32 [1]
    mask: Optional[torch.Tensor]           # uint8 rows x cols/8 (QuEST)
    rows: int
    cols: int
    fmt: int

    @property
    def group(self):
        return GROUP[self.fmt]

    def c_struct(self):
        return fp4_qtensor(self.codes.data_ptr(),
                           self.scales.data_ptr() if self.scales is not None else 0,
                           self.scales_swz.data_ptr() if self.scales_swz is not None else 0,
                           self.tensor_scale.data_ptr(),
                           self.mask.data_ptr() if self.mask is not None else 0,
                           self.rows, self.cols, self.fmt, 0)


def alloc_qtensor(rows, cols, fmt, linear=True, swizzled=True, mask=False, device="cuda"):
    lib = load()
    g = GROUP[fmt]
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=device)
    sc = torch.empty((rows, cols // g), dtype=torch.uint8, device=device) if linear else None
    nswz = lib.fp4_swizzled_scale_bytes(rows, cols // g)
    swz = torch.empty((max(nswz, 1),), dtype=torch.uint8, device=device) if swizzled else None
    ts = torch.empty((1,), dtype=torch.float32, device=device)
    mk = torch.empty((rows, cols // 8), dtype=torch.uint8, device=device) if mask else None
    return QTensor(codes, sc, swz, ts, mk, rows, cols, fmt)


def workspace_size(rows, cols, fmt, rnd, had_block):
    return int(load().fp4_quantize_workspace_size(rows, cols, fmt, rnd, had_block))


def alloc_workspace(nbytes, device="cuda"):
    return torch.empty((max(int(nbytes), 16),), dtype=torch.uint8, device=device)


def quantize(x, fmt, rnd, had_block=0, randomized=False, seed=0, sign_tag=0, tensor_tag=0,
             transpose=False, linear=True, swizzled=True, out=None, ws=None):
    """fp4_quantize of a bf16 CUDA tensor; returns a QTensor."""
    lib = load()
    assert x.dtype == torch.bfloat16 and x.is_cuda and x.dim() == 2 and x.is_contiguous()
    in_rows, in_cols = x.shape
    rows, cols = (in_cols, in_rows) if transpose else (in_rows, in_cols)
    if out is None:
        out = alloc_qtensor(rows, cols, fmt, linear, swizzled, mask=(rnd == QUEST), device=x.device)
    need = workspace_size(rows, cols, fmt, rnd, had_block)
    if ws is None:
        ws = alloc_workspace(need, x.device)
    cs = out.c_struct()
    st = lib.fp4_quantize(_ptr(x), in_rows, in_cols, int(transpose), fmt, rnd, GROUP[fmt],
                          fp4_had(had_block, int(randomized), sign_tag), seed, tensor_tag,
                          ctypes.byref(cs), _ptr(ws), ws.numel(), _stream())
    _check(st, "fp4_quantize")
    return out


def quantize_noalloc(x, fmt, rnd, had_block=0, randomized=False, seed=0, sign_tag=0, tensor_tag=0,
                     transpose=False, out=None):
    """fp4_quantize_noalloc: the same quantisation as quantize(), with the
    library's fixed device scratch instead of a caller workspace (the C call
    allocates nothing; only this binding allocates `out` when not given)."""
    lib = load()
    f = lib.fp4_quantize_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                  ctypes.c_int32, ctypes.c_int32, fp4_had, ctypes.c_uint64, ctypes.c_uint32,
                  ctypes.POINTER(fp4_qtensor), ctypes.c_void_p]
    in_rows, in_cols = x.shape
    rows, cols = (in_cols, in_rows) if transpose else (in_rows, in_cols)
    if out is None:
        out = alloc_qtensor(rows, cols, fmt, mask=(rnd == QUEST), device=x.device)
    cs = out.c_struct()
    st = f(_ptr(x), in_rows, in_cols, int(transpose), fmt, rnd, GROUP[fmt],
           fp4_had(had_block, int(randomized), sign_tag), seed, tensor_tag, ctypes.byref(cs), _stream())
    _check(st, "fp4_quantize_noalloc")
    return out


def requantize(qt, rnd, had_block=0, randomized=False, seed=0, sign_tag=0, tensor_tag=0,
               transpose=True, linear=True, swizzled=True, out=None, ws=None):
    lib = load()
    rows, cols = (qt.cols, qt.rows) if transpose else (qt.rows, qt.cols)
    if out is None:
        out = alloc_qtensor(rows, cols, qt.fmt, linear, swizzled, mask=(rnd == QUEST),
                            device=qt.codes.device)
    need = workspace_size(rows, cols, qt.fmt, rnd, had_block)
    if ws is None:
        ws = alloc_workspace(need, qt.codes.device)
    cin, cout = qt.c_struct(), out.c_struct()
    st = lib.fp4_requantize(ctypes.byref(cin), int(transpose), rnd,
                            fp4_had(had_block, int(randomized), sign_tag), seed, tensor_tag,
                            ctypes.byref(cout), _ptr(ws), ws.numel(), _stream())
    _check(st, "fp4_requantize")
    return out


def dequantize(qt, out_dtype=torch.float32, out=None):
    """fp4_dequantize: the fp32 (or bf16) value of every element of a
    quantised tensor (needs its linear scales)."""
    lib = load()
    f = lib.fp4_dequantize
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(fp4_qtensor), ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p]
    if out is None:
        out = torch.empty((qt.rows, qt.cols), dtype=out_dtype, device=qt.codes.device)
    _check_out(out, (qt.rows, qt.cols), "dequantize out")
    code = {torch.float32: 0, torch.bfloat16: 1}[out.dtype]
    cs = qt.c_struct()
    _check(f(ctypes.byref(cs), _ptr(out), code, _stream()), "fp4_dequantize")
    return out


def quantize_mse_workspace_size(rows, cols):
    lib = load()
    f = lib.fp4_quantize_mse_workspace_size
    f.restype = ctypes.c_size_t
    f.argtypes = [ctypes.c_int64, ctypes.c_int64]
    return f(rows, cols)


def quantize_mse(x, iters=0, linear=True, swizzled=True, out=None, ws=None):
    """fp4_quantize_mse: NVFP4 with MSE-optimal group scales and `iters`
    least-squares tensor-scale updates; returns a QTensor."""
    lib = load()
    f = lib.fp4_quantize_mse
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                  ctypes.POINTER(fp4_qtensor), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    assert x.dtype == torch.bfloat16 and x.is_cuda and x.dim() == 2 and x.is_contiguous()
    rows, cols = x.shape
    if out is None:
        out = alloc_qtensor(rows, cols, NVFP4, linear, swizzled, device=x.device)
    if ws is None:
        ws = alloc_workspace(quantize_mse_workspace_size(rows, cols), x.device)
    cs = out.c_struct()
    _check(f(_ptr(x), rows, cols, int(iters), ctypes.byref(cs), _ptr(ws), ws.numel(), _stream()),
           "fp4_quantize_mse")
    return out


def transpose_square16(qt, linear=True, swizzled=True, out=None):
    """fp4_transpose_square16: the transpose of a square-block quantised tensor."""
    lib = load()
    f = lib.fp4_transpose_square16
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(fp4_qtensor), ctypes.POINTER(fp4_qtensor), ctypes.c_void_p]
    if out is None:
        out = alloc_qtensor(qt.cols, qt.rows, qt.fmt, linear, swizzled, device=qt.codes.device)
    cin, cout = qt.c_struct(), out.c_struct()
    _check(f(ctypes.byref(cin), ctypes.byref(cout), _stream()), "fp4_transpose_square16")
    return out


XFORM_DCT2, XFORM_DST2 = 1, 2


def block_transform(x, kind, block, out=None, ws=None):
    """fp4_block_transform: the orthonormal DCT-II / DST-II of every
    `block`-element block of x's rows (bf16 in, fp32 out)."""
    lib = load()
    lib.fp4_block_transform_workspace_size.restype = ctypes.c_size_t
    lib.fp4_block_transform_workspace_size.argtypes = [ctypes.c_int32]
    f = lib.fp4_block_transform
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                  ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    assert x.dtype == torch.bfloat16 and x.is_cuda and x.dim() == 2 and x.is_contiguous()
    if out is None:
        out = torch.empty(x.shape, dtype=torch.float32, device=x.device)
    assert out.shape == x.shape and out.dtype == torch.float32 and out.is_contiguous(), "out: fp32, x's shape"
    if ws is None:
        ws = alloc_workspace(lib.fp4_block_transform_workspace_size(block), x.device)
    _check(f(_ptr(x), _ptr(out), x.shape[0], x.shape[1], kind, block, _ptr(ws), ws.numel(), _stream()),
           "fp4_block_transform")
    return out


def quantize_f32(y, fmt, rnd, seed=0, tensor_tag=0, linear=True, swizzled=True, out=None, ws=None):
    """fp4_quantize_f32: quantise an already transformed fp32 CUDA tensor."""
    lib = load()
    f = lib.fp4_quantize_f32
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                  ctypes.c_uint64, ctypes.c_uint32, ctypes.POINTER(fp4_qtensor), ctypes.c_void_p, ctypes.c_size_t,
                  ctypes.c_void_p]
    assert y.dtype == torch.float32 and y.is_cuda and y.dim() == 2 and y.is_contiguous()
    rows, cols = y.shape
    if out is None:
        out = alloc_qtensor(rows, cols, fmt, linear, swizzled, mask=(rnd == QUEST), device=y.device)
    if ws is None:
        ws = alloc_workspace(workspace_size(rows, cols, fmt, rnd, 0), y.device)
    cs = out.c_struct()
    _check(f(_ptr(y), rows, cols, fmt, rnd, GROUP[fmt], seed, tensor_tag, ctypes.byref(cs), _ptr(ws), ws.numel(),
             _stream()), "fp4_quantize_f32")
    return out


@dataclass
class FitTensor:
    """MXFP4 with fitted scales: codes, one level per 32 elements, the
    tensor's 256-entry scale table."""
    codes: torch.Tensor
    levels: torch.Tensor
    table: torch.Tensor


def quantize_mx_fit_workspace_size():
    lib = load()
    lib.fp4_quantize_mx_fit_workspace_size.restype = ctypes.c_size_t
    lib.fp4_quantize_mx_fit_workspace_size.argtypes = []
    return int(lib.fp4_quantize_mx_fit_workspace_size())


def quantize_mx_fit(x, had_block=0, ws=None, out=None):
    """fp4_quantize_mx_fit (MXFP4-dagger) of a bf16 CUDA tensor (into `out`,
    a FitTensor of the right shapes, when given)."""
    lib = load()
    lib.fp4_quantize_mx_fit_workspace_size.restype = ctypes.c_size_t
    lib.fp4_quantize_mx_fit_workspace_size.argtypes = []
    f = lib.fp4_quantize_mx_fit
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    assert x.dtype == torch.bfloat16 and x.is_cuda and x.dim() == 2 and x.is_contiguous()
    rows, cols = x.shape
    if out is not None:
        assert (tuple(out.codes.shape) == (rows, cols // 2) and tuple(out.levels.shape) == (rows, cols // 32)
                and tuple(out.table.shape) == (256,) and out.table.dtype == torch.float32
                and out.codes.dtype == torch.uint8 and out.levels.dtype == torch.uint8), "out: wrong shapes or types"
    ft = out if out is not None else FitTensor(torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device),
                                               torch.empty((rows, cols // 32), dtype=torch.uint8, device=x.device),
                                               torch.empty((256,), dtype=torch.float32, device=x.device))
    if ws is None:
        ws = alloc_workspace(lib.fp4_quantize_mx_fit_workspace_size(), x.device)
    _check(f(_ptr(x), rows, cols, had_block, _ptr(ft.codes), _ptr(ft.levels), _ptr(ft.table), _ptr(ws), ws.numel(),
             _stream()), "fp4_quantize_mx_fit")
    return ft


def dequantize_mx_fit(ft, out=None):
    """fp4_dequantize_mx_fit: fp32(E2M1(code) * table[level])."""
    lib = load()
    f = lib.fp4_dequantize_mx_fit
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                  ctypes.c_void_p, ctypes.c_void_p]
    rows, cols = ft.codes.shape[0], ft.codes.shape[1] * 2
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.float32, device=ft.codes.device)
    _check_out(out, (rows, cols), "dequantize_mx_fit out")
    _check(f(_ptr(ft.codes), _ptr(ft.levels), _ptr(ft.table), rows, cols, _ptr(out), _stream()),
           "fp4_dequantize_mx_fit")
    return out


def hadamard(x, block, randomized=False, seed=0, sign_tag=0):
    lib = load()
    y = torch.empty(x.shape, dtype=torch.float32, device=x.device)
    st = lib.fp4_hadamard(_ptr(x), _ptr(y), x.shape[0], x.shape[1],
                          fp4_had(block, int(randomized), sign_tag), seed, _stream())
    _check(st, "fp4_hadamard")
    return y


def swizzle_scales(scales):
    lib = load()
    rows, ng = scales.shape
    out = torch.empty((max(lib.fp4_swizzled_scale_bytes(rows, ng), 1),), dtype=torch.uint8,
                      device=scales.device)
    _check(lib.fp4_swizzle_scales(_ptr(scales), rows, ng, _ptr(out), _stream()), "fp4_swizzle_scales")
    return out


def gemm(A, B, out_dtype=torch.float32, mask=None, inverse_had=0, out=None):
    """fp4_gemm: D = dq(A) dq(B)^T (optionally the Quartet mask + H32^-1 epilogue)."""
    lib = load()
    if out is None:
        out = torch.empty((A.rows, B.rows), dtype=out_dtype, device=A.codes.device)
    _check_out(out, (A.rows, B.rows), "gemm out")
    code = {torch.float32: 0, torch.bfloat16: 1}[out.dtype]
    ca, cb = A.c_struct(), B.c_struct()
    st = lib.fp4_gemm(ctypes.byref(ca), ctypes.byref(cb), _ptr(out), code, _ptr(mask),
                      inverse_had, _stream())
    _check(st, "fp4_gemm")
    return out


RECIPE_QUARTET, RECIPE_QUARTET2, RECIPE_RTN, RECIPE_TETRAJET2, RECIPE_NVIDIA = 0, 1, 2, 3, 4


class fp4_recipe(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("fmt", "fwd_rounding", "fwd_had", "bwd_rounding", "bwd_had",
                                               "bwd_randomized", "mask_epilogue", "out_y", "out_dx",
                                               "out_dw", "w_rounding", "w_reuse")]


class fp4_ctx(ctypes.Structure):
    _fields_ = [("xq", fp4_qtensor), ("wq", fp4_qtensor)]


def recipe(preset):
    r = fp4_recipe()
    _check(load().fp4_recipe_preset(preset, ctypes.byref(r)), "fp4_recipe_preset")
    return r


@dataclass
class LinearCtx:
    """Saved forward context: the quantised X (M x K) and W (N x K)."""
    xq: QTensor
    wq: QTensor
    recipe: fp4_recipe

    def c_struct(self):
        return fp4_ctx(self.xq.c_struct(), self.wq.c_struct())


_DT = {0: torch.float32, 1: torch.bfloat16}


def linear_workspace(r, M, N, K, is_bwd, device="cuda"):
    return alloc_workspace(load().fp4_linear_workspace_size(ctypes.byref(r), M, N, K, int(is_bwd)), device)


def alloc_ctx(r, M, N, K, device="cuda"):
    quest = r.fwd_rounding == QUEST
    return LinearCtx(alloc_qtensor(M, K, r.fmt, mask=quest, device=device),
                     alloc_qtensor(N, K, r.fmt, mask=quest, device=device), r)


def linear_fwd(X, W, r, seed=0, ctx=None, Y=None, ws=None):
    """fp4_linear_fwd: returns (Y, ctx)."""
    lib = load()
    M, K = X.shape
    N = W.shape[0]
    if ctx is None:
        ctx = alloc_ctx(r, M, N, K, X.device)
    if Y is None:
        Y = torch.empty((M, N), dtype=_DT[r.out_y], device=X.device)
    _check_out(Y, (M, N), "linear_fwd Y")
    if ws is None:
        ws = linear_workspace(r, M, N, K, False, X.device)
    c = ctx.c_struct()
    st = lib.fp4_linear_fwd(_ptr(X), _ptr(W), M, N, K, ctypes.byref(r), seed, _ptr(Y), ctypes.byref(c),
                            _ptr(ws), ws.numel(), _stream())
    _check(st, "fp4_linear_fwd")
    return Y, ctx


def linear_bwd(dY, ctx, step_seed, dX=None, dW=None, ws=None, want_dx=True, want_dw=True):
    """fp4_linear_bwd: returns (dX, dW)."""
    lib = load()
    r = ctx.recipe
    M, N = dY.shape
    K = ctx.xq.cols
    if want_dx and dX is None:
        dX = torch.empty((M, K), dtype=_DT[r.out_dx], device=dY.device)
    if want_dw and dW is None:
        dW = torch.empty((N, K), dtype=_DT[r.out_dw], device=dY.device)
    if want_dx:
        _check_out(dX, (M, K), "linear_bwd dX")
    if want_dw:
        _check_out(dW, (N, K), "linear_bwd dW")
    if ws is None:
        ws = linear_workspace(r, M, N, K, True, dY.device)
    c = ctx.c_struct()
    st = lib.fp4_linear_bwd(_ptr(dY), ctypes.byref(c), M, N, K, ctypes.byref(r), step_seed,
                            _ptr(dX if want_dx else None), _ptr(dW if want_dw else None),
                            _ptr(ws), ws.numel(), _stream())
    _check(st, "fp4_linear_bwd")
    return dX, dW


def selftest_e2m1():
    """Mismatching 8-element words between the hardware E2M1 encoder and the
    per-element rounding over all 2^32 fp32 patterns (0 expected)."""
    lib = load()
    lib.fp4_selftest_e2m1.restype = ctypes.c_int
    lib.fp4_selftest_e2m1.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    cnt = torch.zeros((1,), dtype=torch.int64, device="cuda")
    _check(lib.fp4_selftest_e2m1(_ptr(cnt), _stream()), "fp4_selftest_e2m1")
    return int(cnt.item())


def selftest_arith():
    """Mismatch counts of the quantisers' exact division by 6, E8M3
    reciprocal, per-tensor division, E4M3 decoder, E4M3 encoder and MS-EDEN
    pseudo-scale rounding against CUDA's IEEE operations (all 0 expected)."""
    lib = load()
    lib.fp4_selftest_arith.restype = ctypes.c_int
    lib.fp4_selftest_arith.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    cnt = torch.zeros((6,), dtype=torch.int64, device="cuda")
    _check(lib.fp4_selftest_arith(_ptr(cnt), _stream()), "fp4_selftest_arith")
    return [int(v) for v in cnt.cpu()]


def launch_count():
    lib = load()
    lib.fp4_launch_count.restype = ctypes.c_ulonglong
    return int(lib.fp4_launch_count())


def get_last_error():
    return int(load().fp4_get_last_error(_stream()))
