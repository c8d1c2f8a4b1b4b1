"""Seeded synthetic inputs (bf16) for tests, the smoke check and the bench.

This module holds no arithmetic of the quantisation method: it only draws
numbers and rounds them to bf16.  It is the one module both the CUDA path's
callers and the oracle's callers share.

Recipes (the pages' workloads -- LLM activations, weights and gradients --
are replaced by these distributions):
* Gaussian weights N(0, 0.02^2) and Gaussian activations N(0, 1);
* activations with outlier channels: ceil(1% of K) columns, chosen by a
  seeded permutation, multiplied by 20;
* heavy-tailed activations: Student-t with nu = 3 divided by the tensor's
  empirical RMS; heavy-tailed gradients: 1e-3 * Student-t(3), unscaled;
* quantizer sweep tensors: N(0, 1) plus 0.1% of elements (seeded
  positions) multiplied by 50.
All generation is numpy PCG64 in float32, then round-to-nearest-even to bf16.
"""
import numpy as np


def rng(seed, stream=0):
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([0xF4F4, int(seed), int(stream)])))


def f32_to_bf16_bits(x):
    """Round-to-nearest-even float32 -> bf16 bit patterns (uint16)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((b >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    out = ((b + r) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def gaussian(shape, std, seed, stream=0):
    x = rng(seed, stream).standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return f32_to_bf16_bits(x)


def student_t(shape, seed, stream=0, nu=3.0, scale=1.0, unit_rms=False):
    g = rng(seed, stream)
    z = g.standard_normal(shape, dtype=np.float32)
    chi = g.standard_gamma(nu / 2.0, size=shape, dtype=np.float32) * np.float32(2.0)
    x = z / np.sqrt(chi / np.float32(nu))
    if unit_rms:
        x /= np.float32(np.sqrt(np.mean(np.square(x, dtype=np.float64))))
    if scale != 1.0:
        x *= np.float32(scale)
    return f32_to_bf16_bits(x)


def outlier_channels(shape, seed, stream=0, frac=0.01, factor=20.0):
    rows, cols = shape
    x = rng(seed, stream).standard_normal(shape, dtype=np.float32)
    n = int(np.ceil(frac * cols))
    cols_sel = rng(seed, stream + 1000).permutation(cols)[:n]
    x[:, cols_sel] *= np.float32(factor)
    return f32_to_bf16_bits(x)


def outlier_elements(shape, seed, stream=0, frac=0.001, factor=50.0):
    x = rng(seed, stream).standard_normal(shape, dtype=np.float32)
    flat = x.reshape(-1)
    n = int(round(frac * flat.size))
    pos = rng(seed, stream + 1000).choice(flat.size, size=n, replace=False)
    flat[pos] *= np.float32(factor)
    return f32_to_bf16_bits(x)


def grid_values(shape, seed, stream=0, step=0.125, kmax=48):
    """Values k * step for uniform random integers |k| <= kmax: exact in bf16
    and so coarse that many 16-element groups have two equally good scales
    (tie-breaking and last-bit cases)."""
    k = rng(seed, stream).integers(-kmax, kmax + 1, size=shape)
    return f32_to_bf16_bits((k * step).astype(np.float32))


# ------------------------------------------------------- named workloads ----
def linear_rtn_small(seed=0):
    """Single NVFP4 RTN forward linear: X 256x512 ~N(0,1), W 512x512 ~N(0,0.02^2)."""
    return {"X": gaussian((256, 512), 1.0, seed, 0), "W": gaussian((512, 512), 0.02, seed, 1)}


def linear_quartet(M=4096, N=2048, K=2048, seed=1):
    """Quartet MXFP4 layer: X with 1% outlier channels x20, W ~N(0,0.02^2),
    dY ~N(0,1e-3^2)."""
    return {"X": outlier_channels((M, K), seed, 0), "W": gaussian((N, K), 0.02, seed, 1),
            "dY": gaussian((M, N), 1e-3, seed, 2)}


def linear_quartet2(M=8192, N=8192, K=2048, seed=2):
    """Quartet II NVFP4 layer: X Student-t(3) at unit RMS, W ~N(0,0.02^2),
    dY = 1e-3 * Student-t(3)."""
    return {"X": student_t((M, K), seed, 0, unit_rms=True), "W": gaussian((N, K), 0.02, seed, 1),
            "dY": student_t((M, N), seed, 2, scale=1e-3)}


LLAMA3_8B_LAYERS = (("qkv", 4096, 6144), ("o", 4096, 4096), ("gate_up", 4096, 28672),
                    ("down", 14336, 4096))


def quantizer_sweep(n_elems, seed=7, row=4096):
    """Quantizer-only sweep tensor: rows of 4096, N(0,1) plus 0.1% x50."""
    return outlier_elements((n_elems // row, row), seed, 0)
