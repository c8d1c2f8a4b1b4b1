"""Block Hadamard transforms: deterministic H_g and the randomized RHT_g.

Test infrastructure only (see ``oracle/__init__.py``).

Quartet page, "The Hadamard Transform": the normalised g x g Hadamard matrix
is built by the Sylvester recursion H_2k = H_2 (x) H_k with the 1/sqrt(g)
normalisation, so H_g is orthogonal and symmetric; the transform multiplies
each g-block of a vector (along the GEMM's inner dimension) by H_g.  The
forward pass uses it as is; the backward pass randomises it with random sign
flips (Quartet page; Quartet II page, MS-EDEN Step 1, one sign pattern per
tensor shared by every chunk and by both operands of a GEMM).

Readings (the pages leave these open):
* fp32 evaluation order: the in-place fast Walsh-Hadamard butterflies
  (a, b) -> (a + b, a - b) on index pairs (i, i + h), i & h == 0, for
  h = 1, 2, ..., g/2 (Sylvester natural order), then one multiply by
  c_g = fp32(1/sqrt(g)).
* RHT = H_g . diag(d): the sign flip is applied to the input, once.  The
  Quartet page's second flip after H_g is dropped: every quantizer here is
  symmetric under a sign change of an element (and the GEMM operands share
  the signs), so it would cancel exactly.
"""
import numpy as np

from . import philox

F32 = np.float32


def sylvester(g):
    """Unnormalised +-1 Sylvester-Hadamard matrix of order g (fp64), by the
    Kronecker recursion H_2k = H_2 (x) H_k."""
    h = np.array([[1.0]])
    h2 = np.array([[1.0, 1.0], [1.0, -1.0]])
    while h.shape[0] < g:
        h = np.kron(h2, h)
    return h


def hadamard_scale(g):
    """c_g = fp32(1/sqrt(g)), rounded once from fp64."""
    return F32(1.0 / np.sqrt(float(g)))


def fwht_f32(x, g):
    """fp32 block Walsh-Hadamard transform of the last axis in blocks of g,
    including the c_g normalisation (the butterfly order in the module doc)."""
    x = np.asarray(x, dtype=F32)
    n = x.shape[-1]
    assert n % g == 0
    lead = x.shape[:-1]
    y = x.reshape(-1, n // g, g).copy()
    h = 1
    while h < g:
        v = y.reshape(y.shape[0], y.shape[1], g // (2 * h), 2, h)
        a = v[:, :, :, 0, :].copy()
        b = v[:, :, :, 1, :].copy()
        v[:, :, :, 0, :] = (a + b).astype(F32)
        v[:, :, :, 1, :] = (a - b).astype(F32)
        h *= 2
    y = (y * hadamard_scale(g)).astype(F32)
    return y.reshape(lead + (n,))


def block_transform(x, had_block, randomized, seed=0, sign_tag=0):
    """Apply H_g (randomized=False) or RHT_g (randomized=True) along the last
    axis of fp32 ``x`` in blocks of ``had_block``; ``had_block == 0`` is the
    identity."""
    x = np.asarray(x, dtype=F32)
    if had_block == 0:
        return x.copy()
    if randomized:
        d = philox.rht_signs(seed, sign_tag, had_block)
        n = x.shape[-1]
        x = (x.reshape(x.shape[:-1] + (n // had_block, had_block)) * d).astype(F32)
        x = x.reshape(x.shape[:-2] + (n,))
    return fwht_f32(x, had_block)


def block_transform_f64(x, had_block, randomized, seed=0, sign_tag=0):
    """The same transform as an exact fp64 matrix product (for references)."""
    x = np.asarray(x, dtype=np.float64)
    if had_block == 0:
        return x.copy()
    n = x.shape[-1]
    hm = sylvester(had_block) / np.sqrt(float(had_block))
    if randomized:
        d = philox.rht_signs(seed, sign_tag, had_block).astype(np.float64)
        hm = hm * d[None, :]          # H . diag(d)
    xb = x.reshape(x.shape[:-1] + (n // had_block, had_block))
    return (xb @ hm.T).reshape(x.shape)


def inverse_block_h_f64(y, had_block):
    """H_g^-1 = H_g (symmetric and orthogonal), applied per block in fp64."""
    return block_transform_f64(y, had_block, randomized=False)
