"""Counter-based random numbers: Philox4x32-10.

Test infrastructure only (see ``oracle/__init__.py``).

The pages require seeded randomness for the randomized Hadamard signs
(Quartet page, "The Hadamard Transform": random seed xi; Quartet II page,
MS-EDEN Step 1: omega_RHT) and for stochastic rounding (Quartet II page,
Step 3 and MS-EDEN Step 4: omega_SR) but name no generator.  Both the oracle
and the CUDA path use Philox4x32 with 10 rounds, written here from its
published definition (Salmon, Moraes, Dror, Shaw, "Parallel random numbers:
as easy as 1, 2, 3", SC'11): a 4x32-bit counter, a 2x32-bit key, each round
    (hi0, lo0) = mulhilo(0xD2511F53, c0);  (hi1, lo1) = mulhilo(0xCD9E8D57, c2)
    c <- (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0)
and the key bumped by (0x9E3779B9, 0xBB67AE85) between rounds.

Stream layout (a reading, the pages give none): key = the 64-bit seed,
counter = (q_lo, q_hi, purpose tag, tensor tag) with q = index >> 2; the
value for ``index`` is word ``index & 3`` of that block, so four
consecutive indices share one Philox call.
"""
import numpy as np

M0 = np.uint64(0xD2511F53)
M1 = np.uint64(0xCD9E8D57)
W0 = np.uint64(0x9E3779B9)
W1 = np.uint64(0xBB67AE85)
MASK32 = np.uint64(0xFFFFFFFF)

TAG_SR_ELEM = 1    # element-wise stochastic rounding of FP4 codes
TAG_SR_SCALE = 2   # stochastic rounding of E4M3 group scales (MS-EDEN)
TAG_RHT_SIGN = 3   # random signs of the randomized Hadamard transform


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Vectorised Philox4x32-10.  All inputs are uint32-valued arrays (or
    scalars) broadcast together; returns four uint32 arrays."""
    c0, c1, c2, c3 = (np.asarray(c, dtype=np.uint64) & MASK32 for c in (c0, c1, c2, c3))
    k0 = np.asarray(k0, dtype=np.uint64) & MASK32
    k1 = np.asarray(k1, dtype=np.uint64) & MASK32
    c0, c1, c2, c3, k0, k1 = np.broadcast_arrays(c0, c1, c2, c3, k0, k1)
    c0, c1, c2, c3, k0, k1 = (c.copy() for c in (c0, c1, c2, c3, k0, k1))
    for r in range(10):
        if r > 0:
            k0 = (k0 + W0) & MASK32
            k1 = (k1 + W1) & MASK32
        p0 = M0 * c0
        p1 = M1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & MASK32
        c0, c1, c2, c3 = (hi1 ^ c1 ^ k0) & MASK32, lo1, (hi0 ^ c3 ^ k1) & MASK32, lo0
    return tuple(c.astype(np.uint32) for c in (c0, c1, c2, c3))


def split_seed(seed):
    """64-bit seed (scalar or array) -> (low word, high word)."""
    if np.ndim(seed) == 0:
        seed = int(seed) & 0xFFFFFFFFFFFFFFFF
        return seed & 0xFFFFFFFF, seed >> 32
    seed = np.asarray(seed, dtype=np.uint64)
    return seed & MASK32, seed >> np.uint64(32)


def words(seed, index, tag, tensor_tag):
    """32-bit random word for each (non-negative) ``index`` of one stream;
    ``seed`` may be an array broadcast against ``index``."""
    index = np.asarray(index, dtype=np.uint64)
    q = index >> np.uint64(2)
    k0, k1 = split_seed(seed)
    out = philox4x32_10(q & MASK32, q >> np.uint64(32), np.uint64(tag),
                        np.uint64(tensor_tag & 0xFFFFFFFF), k0, k1)
    w = np.stack(out, axis=-1)
    lane = np.broadcast_to((index & np.uint64(3)).astype(np.int64), w.shape[:-1])
    return np.take_along_axis(w, lane[..., None], axis=-1)[..., 0]


def uniform(seed, index, tag, tensor_tag):
    """u = (word >> 8) * 2^-24: uniform on the 2^24 multiples of 2^-24 in [0,1)."""
    w = words(seed, index, tag, tensor_tag).astype(np.uint64)
    return (w >> np.uint64(8)).astype(np.float64) * 2.0 ** -24


def rht_signs(seed, sign_tag, g):
    """Random +-1 diagonal of the randomized Hadamard transform: d_j = -1
    iff bit 31 of word j of the (seed, TAG_RHT_SIGN, sign_tag) stream.  One
    pattern of length g serves every g-block of a tensor (Quartet II page,
    MS-EDEN Step 1: the same seed for all chunks) and both operands of a
    GEMM that share ``seed`` and ``sign_tag``."""
    w = words(seed, np.arange(g, dtype=np.uint64), TAG_RHT_SIGN, sign_tag)
    return np.where(w >> np.uint32(31), -1.0, 1.0).astype(np.float32)
