"""CPU checks of the boundary: the C-ABI library loads and exports every
function include/*.h declares; host-side helpers answer without a GPU."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "fp4_microscaled_quantized_b200", "libfp4_b200.so")


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"\b(fp4_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        from fp4_microscaled_quantized_b200 import build
        build.build()
    return ctypes.CDLL(LIB)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "fp4_quantize" in names and "fp4_hadamard" in names
    for n in names:
        assert hasattr(lib, n), n


def test_host_helpers_without_gpu(lib):
    lib.fp4_quantize_workspace_size.restype = ctypes.c_size_t
    lib.fp4_quantize_workspace_size.argtypes = [ctypes.c_int64] * 2 + [ctypes.c_int32] * 3
    lib.fp4_swizzled_scale_bytes.restype = ctypes.c_size_t
    lib.fp4_swizzled_scale_bytes.argtypes = [ctypes.c_int64] * 2
    lib.fp4_status_string.restype = ctypes.c_char_p
    assert lib.fp4_quantize_workspace_size(128, 512, 0, 0, 32) == 0          # MXFP4: no pass
    assert lib.fp4_quantize_workspace_size(128, 512, 1, 0, 0) == 256         # amax word
    eden = lib.fp4_quantize_workspace_size(128, 512, 1, 4, 128)
    assert eden >= 256 + 128 * 32 * 2 + 128 * 4 * 4
    assert lib.fp4_swizzled_scale_bytes(300, 10) == 3 * 3 * 512
    assert lib.fp4_status_string(2) == b"unsupported combination"
    lib.fp4_quantize_mse_workspace_size.restype = ctypes.c_size_t
    lib.fp4_quantize_mse_workspace_size.argtypes = [ctypes.c_int64] * 2
    # amax word + one float64 pair per 8192 elements, rounded up to 256 bytes
    assert lib.fp4_quantize_mse_workspace_size(64, 256) == 256 + 256
    assert lib.fp4_quantize_mse_workspace_size(10240, 4096) == 256 + 5120 * 16
    assert lib.fp4_quantize_mse_workspace_size(0, 256) == 256
    assert lib.fp4_quantize_mse_workspace_size(64, 48) == 0                 # cols not a multiple of 32


def test_product_path_does_not_import_oracle():
    pkg = os.path.join(ROOT, "fp4_microscaled_quantized_b200")
    for path in glob.glob(os.path.join(pkg, "**", "*.py"), recursive=True):
        src = open(path).read()
        assert not re.search(r"^\s*(from|import)\s+oracle", src, flags=re.M), path
    for path in glob.glob(os.path.join(pkg, "csrc", "*")):
        assert "oracle" not in open(path).read(), path
