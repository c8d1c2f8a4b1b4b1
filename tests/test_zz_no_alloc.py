"""fp4_quantize_noalloc: quantisation for callers that cannot allocate device
memory when they quantise (a framework or serving engine that owns all device
memory, a plugin handed only its inputs and outputs, a loop where cudaMalloc's
possible device synchronisation is not acceptable).  The call takes no
workspace and allocates nothing; its scratch is a fixed 4 MiB array inside the
library.  Its results must equal fp4_quantize's bit for bit, on consecutive
calls (the shared array keeps the previous call's contents, and the part that
must start at zero is cleared inside each call).

This file is collected last on purpose, so a failure here never hides the
results of the other tests."""
import numpy as np
import pytest
import torch

from fp4_microscaled_quantized_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _same(a, b):
    torch.cuda.synchronize()
    for name in ("codes", "scales", "scales_swz", "tensor_scale"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    if a.mask is not None:
        assert torch.equal(a.mask, b.mask)


@pytest.mark.parametrize("fmt,rnd,had,transpose", [
    (1, 4, 128, False),     # NVFP4 MS-EDEN: amax word + pseudo-scales + EDEN factors in the scratch
    (1, 4, 128, True),
    (1, 2, 0, False),       # NVFP4 Four-Over-Six: amax word in the scratch
    (0, 3, 32, False),      # MXFP4 SR: no scratch at all
    (1, 5, 0, False),       # NVFP4 16 x 16 square blocks: one maximum per block in the scratch
    (1, 5, 0, True),
])
def test_noalloc_matches_regular_quantize_twice(cuda_lib, fmt, rnd, had, transpose):
    first = _dev(syn.student_t((1024, 2048), seed=21, unit_rms=True))
    # different data with a far smaller amax and block maxima, so anything
    # left in the shared scratch by the first call would change the second
    second = _dev(syn.gaussian((1024, 2048), 0.02, seed=22))
    for k, x in enumerate((first, second)):
        ref = cuda_lib.quantize(x, fmt, rnd, had, randomized=True, seed=5 + k, tensor_tag=3,
                                transpose=transpose)
        got = cuda_lib.quantize_noalloc(x, fmt, rnd, had, randomized=True, seed=5 + k, tensor_tag=3,
                                        transpose=transpose)
        _same(got, ref)
    assert cuda_lib.get_last_error() == 0


def test_noalloc_rejects_tensors_beyond_the_scratch(cuda_lib):
    x = torch.zeros((8192, 4096), dtype=torch.bfloat16, device="cuda")   # MS-EDEN needs ~5.2 MB
    n0 = cuda_lib.launch_count()
    with pytest.raises(cuda_lib.Fp4Error) as e:
        cuda_lib.quantize_noalloc(x, 1, 4, 128, randomized=True)
    assert e.value.status == 4                                           # FP4_ERR_WORKSPACE
    assert cuda_lib.launch_count() == n0                                 # nothing launched
