"""The per-unit algorithmic figures behind bench.py's roofline numbers, on the
CPU: bytes per quantised element of each quantiser call and the layer set's
flops."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_quantiser_bytes_per_element():
    # Four-Over-Six: amax read 2 + bf16 read 2 + codes 0.5 + one scale copy 1/16
    assert bench.quant_bytes_per_elem("fos") == pytest.approx(4.5625)
    # MS-EDEN from bf16: 2 + 0.5 + 1/16 + pseudo-scales 2 x 2/16 + EDEN factors 2 x 4/128
    assert bench.quant_bytes_per_elem("eden") == pytest.approx(2.875)
    # MS-EDEN re-quantisation: FP4 in (0.5 + 1/16) and out, same pseudo-scale and factor traffic
    assert bench.quant_bytes_per_elem("eden_requant") == pytest.approx(1.4375)
    with pytest.raises(ValueError):
        bench.quant_bytes_per_elem("rtn")


def test_layer_set_work():
    """Llama-3-8B-shaped layer set at 16384 tokens: sum N K = 218.1 M weights,
    6 M sum N K = 21.44 TFLOP per fwd+bwd step."""
    nk = sum(K * N for _, K, N in bench.LAYERS)
    assert nk == 4096 * 6144 + 4096 * 4096 + 4096 * 28672 + 14336 * 4096
    assert 6.0 * bench.M_TOKENS * nk / 1e12 == pytest.approx(21.44, rel=1e-3)


def test_sweep_bytes_per_element():
    from fp4_microscaled_quantized_b200 import api
    assert bench.sweep_bytes_per_elem(api, api.NVFP4, api.RTN, 0) == pytest.approx(4.5625)
    assert bench.sweep_bytes_per_elem(api, api.MXFP4, api.QUEST, 32) == pytest.approx(2.53125 + 0.125)
    assert bench.sweep_bytes_per_elem(api, api.NVFP4, api.MS_EDEN, 128) == pytest.approx(2.875)
    assert bench.sweep_bytes_per_elem(api, api.NVFP4, "mse2", 0) == pytest.approx(2 + 3 * 2.5625)
    # transform (bf16 read, fp32 write) + fp32 quantiser (NVFP4: amax read, read, codes, scales)
    assert bench.sweep_bytes_per_elem(api, api.NVFP4, ("xform", "dct2", 128), 128) == pytest.approx(14.5625)
    assert bench.sweep_bytes_per_elem(api, api.MXFP4, ("xform", "dst2", 256), 256) == pytest.approx(10.53125)
    # MXFP4 with fitted scales: range pass + quantise pass
    assert bench.sweep_bytes_per_elem(api, api.MXFP4, ("fit",), 0) == pytest.approx(4.53125)


def test_sweep_cases_are_unique_and_cover_the_forward_only_variants():
    from fp4_microscaled_quantized_b200 import api
    names = [c[0] for c in bench.sweep_cases(api)]
    assert len(names) == len(set(names))
    for n in ("nvfp4-rtn-dct2-k32", "nvfp4-rtn-dct2-k128", "mxfp4-rtn-dst2-k256", "mxfp4-fit-h0", "mxfp4-fit-h32",
              "nvfp4-mse-i0-h0", "nvfp4-eden-h128"):
        assert n in names
