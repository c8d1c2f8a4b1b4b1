"""Number formats of micro-scaled FP4: E2M1 elements, E4M3 / E8M0 scales,
the E8M3 pseudo-scale, fixed pairwise sums and the packed storage layout.

Test infrastructure only (see ``oracle/__init__.py``).

Sources:
* Quartet II page, "NVFP4 Format and Standard Stochastic Rounding": the
  E2M1 value set {0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6}, one E4M3 scale
  per 16 elements, one FP32 tensor scale, dequantisation
  x = x_fp4 * x_fp8 * x_fp32, the E4M3 maximum 448.
* Bridging-the-Gap page (MXFP4 / NVFP4 formats): MXFP4 = E2M1 with one
  power-of-two E8M0 scale per 32 elements; the E2M1 dead zone |v| < 0.25
  rounds to zero.
* Quartet II page, "Post hoc range alignment kernel design": pseudo-scales
  with three mantissa bits and an extended exponent range ("E8M3"), stored in
  BF16.

Every rounding here is written as its plain definition (nearest point of an
explicit value table, ties to the even code; stochastic rounding with the
exact interpolation probability) so a reader can check it by eye.
"""
import numpy as np

F32 = np.float32

# E2M1 magnitudes indexed by the 3 low bits of the code (bit 3 is the sign).
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
E2M1_MAX = 6.0

_CHUNK = 1 << 21


def _chunked(fn, *arrays):
    """Apply an elementwise ``fn`` over flat chunks (bounds temporary memory)."""
    shape = arrays[0].shape
    flat = [np.ascontiguousarray(a).reshape(-1) for a in arrays]
    out = None
    n = flat[0].size
    for s in range(0, n, _CHUNK):
        r = fn(*[a[s:s + _CHUNK] for a in flat])
        if out is None:
            out = np.empty(n, dtype=r.dtype)
        out[s:s + _CHUNK] = r
    if out is None:
        out = fn(*[a[:0] for a in flat])
    return out.reshape(shape)


def _nearest_index(a, table):
    """Index of the nearest entry of the increasing ``table`` to each a >= 0;
    a tie between two neighbours goes to the even index (round half to even
    on the code); values beyond the last entry saturate to it."""
    a = np.minimum(a.astype(np.float64), table[-1])   # saturate first
    d = np.abs(a[:, None] - table[None, :])
    idx = np.argmin(d, axis=1)                      # lowest index among ties
    nxt = np.minimum(idx + 1, table.size - 1)
    dmin = d[np.arange(a.size), idx]
    dnxt = d[np.arange(a.size), nxt]
    tie = (dnxt == dmin) & (nxt != idx)
    return np.where(tie & (idx % 2 == 1), nxt, idx)


def rtn_e2m1(v):
    """Round-to-nearest E2M1 code of each float32 ``v`` (ties to even code,
    saturating at +-6, -0 encoded as +0). Returns uint8 codes 0..15."""
    v = np.asarray(v, dtype=F32)
    if np.isnan(v).any():
        raise ValueError("rtn_e2m1: NaN input")

    def f(x):
        mag = _nearest_index(np.abs(x), E2M1_GRID).astype(np.uint8)
        neg = (x < 0) & (mag != 0)
        return (mag | (neg.astype(np.uint8) << 3)).astype(np.uint8)

    return _chunked(f, v)


def decode_e2m1(codes):
    """E2M1 code -> float32 value."""
    codes = np.asarray(codes, dtype=np.uint8)
    mag = E2M1_GRID[codes & 7]
    return np.where(codes & 8, -mag, mag).astype(F32)


def sr_e2m1(v, u):
    """Stochastic rounding of float32 ``v`` onto the E2M1 grid: between the
    two neighbouring grid points lo <= |v| <= hi it returns hi with
    probability (|v|-lo)/(hi-lo), i.e. iff u < (|v|-lo)/(hi-lo) for the
    uniform u in [0,1).  |v| >= 6 saturates to 6.  (Quartet II page, "NVFP4
    Format and Standard Stochastic Rounding", Step 3.)"""
    v = np.asarray(v, dtype=F32)
    u = np.asarray(u, dtype=np.float64)
    if np.isnan(v).any():
        raise ValueError("sr_e2m1: NaN input")

    def f(x, uu):
        a = np.abs(x).astype(np.float64)
        a = np.minimum(a, E2M1_MAX)
        lo_i = np.searchsorted(E2M1_GRID, a, side="right") - 1
        lo_i = np.minimum(lo_i, 7)
        hi_i = np.minimum(lo_i + 1, 7)
        lo = E2M1_GRID[lo_i]
        hi = E2M1_GRID[hi_i]
        width = np.where(hi_i > lo_i, hi - lo, 1.0)
        frac = np.where(hi_i > lo_i, (a - lo) / width, 0.0)
        mag = np.where(uu < frac, hi_i, lo_i).astype(np.uint8)
        neg = (x < 0) & (mag != 0)
        return (mag | (neg.astype(np.uint8) << 3)).astype(np.uint8)

    return _chunked(f, v, u)


# ---------------------------------------------------------------- E4M3 ----
def _e4m3_table():
    vals = []
    for code in range(127):          # 0x7F is NaN in E4M3; 0x7E = 448 is max
        e, m = code >> 3, code & 7
        if e == 0:
            vals.append(m * 2.0 ** -9)
        else:
            vals.append((1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(vals, dtype=np.float64)


E4M3_VALUES = _e4m3_table()          # strictly increasing, index == code
E4M3_MAX = 448.0
E4M3_MIN_NORMAL = 2.0 ** -6


def e4m3_value(codes):
    return E4M3_VALUES[np.asarray(codes, dtype=np.int64)]


def rtn_e4m3(t):
    """Round-to-nearest-even of non-negative float32 ``t`` to an E4M3 code,
    saturating at 448 (the E4M3 maximum named on the Quartet II page)."""
    t = np.asarray(t, dtype=F32)
    if np.isnan(t).any() or (t < 0).any():
        raise ValueError("rtn_e4m3: needs finite non-negative input")
    return _chunked(lambda x: _nearest_index(x, E4M3_VALUES).astype(np.uint8), t)


def sr_e4m3(t, u):
    """Stochastic rounding of non-negative float32 ``t`` to E4M3 (Quartet II
    page, MS-EDEN Step 4).  Values below the smallest normal E4M3 value 2^-6
    are rounded to nearest instead ("not stochastically rounding underflowing
    FP8 values", Quartet II page, Unbiasedness Verification); t >= 448
    saturates to 448."""
    t = np.asarray(t, dtype=F32)
    u = np.asarray(u, dtype=np.float64)
    if np.isnan(t).any() or (t < 0).any():
        raise ValueError("sr_e4m3: needs finite non-negative input")

    def f(x, uu):
        a = x.astype(np.float64)
        rtn = _nearest_index(x, E4M3_VALUES)
        lo_i = np.clip(np.searchsorted(E4M3_VALUES, a, side="right") - 1, 0, 126)
        hi_i = np.minimum(lo_i + 1, 126)
        lo = E4M3_VALUES[lo_i]
        hi = E4M3_VALUES[hi_i]
        width = np.where(hi_i > lo_i, hi - lo, 1.0)
        frac = np.where(hi_i > lo_i, (a - lo) / width, 0.0)
        sr = np.where(uu < frac, hi_i, lo_i)
        out = np.where(a < E4M3_MIN_NORMAL, rtn, sr)
        out = np.where(a >= E4M3_MAX, 126, out)
        return out.astype(np.uint8)

    return _chunked(f, t, u)


# ---------------------------------------------------------------- E8M0 ----
def e8m0_value(codes):
    """E8M0 scale code c -> 2^(c-127) (fp64, exact)."""
    return np.ldexp(1.0, np.asarray(codes, dtype=np.int64) - 127)


# ---------------------------------------------------------------- E8M3 ----
def e8m3_round(t):
    """Round positive float32 ``t`` to three fractional mantissa bits
    (ties to even) keeping the full fp32 exponent range: the pseudo-scale
    format of the post hoc range alignment (Quartet II page, Figures 7-8).
    Below 2^-126 the grid step stays 2^-129 (the fp32 subnormal binade).
    The result is exactly representable in BF16."""
    t = np.asarray(t, dtype=F32).astype(np.float64)
    if (t < 0).any() or np.isnan(t).any():
        raise ValueError("e8m3_round: needs finite non-negative input")
    _, ex = np.frexp(t)              # t = m * 2^ex, m in [0.5, 1)
    e = np.maximum(ex - 1, -126)     # floor(log2 t), clamped
    step = np.ldexp(1.0, e - 3)
    q = np.rint(t / step) * step     # np.rint rounds half to even
    q = np.where(t == 0, 0.0, q)
    return q.astype(F32)


# ------------------------------------------------------- fixed sum order ----
def pairwise_sum(a):
    """Sum along the last axis (a power-of-two length) as a fixed pairwise
    tree in float32: level 0 adds elements (2i, 2i+1), the next level adds
    adjacent pair sums, and so on."""
    a = np.asarray(a, dtype=F32)
    n = a.shape[-1]
    assert n & (n - 1) == 0, "pairwise_sum needs a power-of-two length"
    while a.shape[-1] > 1:
        a = (a[..., 0::2] + a[..., 1::2]).astype(F32)
    return a[..., 0]


# ---------------------------------------------------------- storage ----
def pack_codes(codes):
    """(rows, cols) codes -> (rows, cols/2) bytes; element 2j in the low
    nibble, element 2j+1 in the high nibble."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)


def unpack_codes(packed):
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = packed & 0xF
    out[..., 1::2] = packed >> 4
    return out


def pack_mask(mask):
    """(rows, cols) bool -> (rows, cols/8) bytes, element 8b+j in bit j."""
    return np.packbits(np.asarray(mask, dtype=bool), axis=-1, bitorder="little")


def unpack_mask(packed, cols):
    return np.unpackbits(np.asarray(packed, dtype=np.uint8), axis=-1,
                         bitorder="little")[..., :cols].astype(bool)


def f32_bits(x):
    return np.asarray(x, dtype=F32).view(np.uint32)
