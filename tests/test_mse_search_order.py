"""The visiting order and skip rules of the GPU group step of the MSE scale
search, modelled on the oracle's per-candidate errors, select exactly the
exhaustive scan's scale (the oracle's definition: every E4M3 code 1..126,
smallest fp32 error, ties to the larger code).

The kernel evaluates a seed near the AbsMax scale, then seed + k and
seed - k for k = 1, 2, ...; it skips a candidate whose top-element error term
exceeds the best error so far (the group error is a round-to-nearest sum of
non-negative terms, never below one of them), and stops the downward scan at
a skipped candidate whose scale is unusable or satisfies fp32(6 d) <= |top|
(the top term is then a clipping error that only grows as d shrinks).  These
tests check that argument on inputs chosen to stress it: exact ties, groups
with one non-zero value, tensor scales under which small codes give unusable
(sub-normal reciprocal) scales and large codes overflow."""
import numpy as np
import pytest

from fp4_microscaled_quantized_b200 import synthetic as syn
from oracle import formats as fm
from oracle import quant as qn

F32 = np.float32


def _candidate_tables(G, s_T):
    """Per group and code: the fp32 group error and the top element's term."""
    n = G.shape[0]
    d = (fm.E4M3_VALUES[:127].astype(F32) * F32(s_T)).astype(F32)
    inv = (F32(1.0) / d).astype(F32)
    ok = np.isfinite(inv) & (d > 0)
    gm = np.max(np.abs(G), axis=1).astype(F32)
    xt = G[np.arange(n), np.argmax(np.abs(G) == gm[:, None], axis=1)]
    err = np.full((n, 127), np.nan, dtype=F32)
    top = np.full((n, 127), np.nan, dtype=F32)
    with np.errstate(over="ignore", invalid="ignore"):
        for c in range(1, 127):
            dd = np.full(n, d[c], dtype=F32)
            codes, _, _ = qn._encode_rtn(G[None], dd[None])
            err[:, c] = qn._sse(G[None], codes, dd[None])[0]
            v = (xt * (inv[c] if ok[c] else F32(0.0))).astype(F32)
            q = fm.decode_e2m1(fm.rtn_e2m1(v) if ok[c] else np.zeros(n, np.uint8)).astype(F32)
            e = (xt - (q * d[c]).astype(F32)).astype(F32)
            top[:, c] = (e * e).astype(F32)
    return d, inv, ok, gm, xt, err, top


def _kernel_order(G, s_T):
    d, inv, ok, gm, xt, err, top = _candidate_tables(G, s_T)
    n = G.shape[0]
    with np.errstate(over="ignore", invalid="ignore"):
        i6 = F32(F32(1.0) / F32(F32(6.0) * F32(s_T)))
        seed = np.clip(fm.rtn_e4m3(np.nan_to_num((gm * i6).astype(F32), nan=448.0)).astype(np.int64), 1, 126)
    on = gm > 0
    best = np.full(n, np.inf, dtype=F32)
    bc = np.zeros(n, dtype=np.int64)
    rows = np.arange(n)

    def consider(mask, c):
        e = err[rows, c]
        win = mask & ((e < best) | ((e == best) & (c > bc)))
        best[win] = e[win]
        bc[win] = c[win]

    consider(on, seed)
    dn = on.copy()
    for k in range(1, 126):
        up, lo = seed + k, seed - k
        upm = on & (up <= 126)
        dn &= lo >= 1
        upc, loc = np.minimum(up, 126), np.maximum(lo, 1)
        consider(upm & ~(top[rows, upc] > best), upc)
        skip = top[rows, loc] > best
        stop = ~ok[loc] | ((F32(6.0) * d[loc]).astype(F32) <= np.abs(xt))
        consider(dn & ~skip, loc)
        dn &= ~(skip & stop)
    return np.where(on, bc, 0)


def _check(x, s_T):
    G = np.asarray(x, dtype=F32).reshape(-1, 16)
    with np.errstate(all="ignore"):                           # overflowing candidate scales
        ref = qn.mse_group_scales(G.reshape(1, -1, 16), s_T).reshape(-1)
        got = _kernel_order(G, s_T)
    np.testing.assert_array_equal(got, ref.astype(np.int64))


@pytest.mark.parametrize("kind", ["t3", "gauss", "outliers", "grid"])
@pytest.mark.parametrize("scale_factor", [1.0, 1.37, 0.61, 4.0])
def test_kernel_search_order_matches_exhaustive_scan(kind, scale_factor):
    shape = (8, 512)
    bits = {"t3": lambda: syn.student_t(shape, 5, scale=0.02), "gauss": lambda: syn.gaussian(shape, 1.0, 6),
            "outliers": lambda: syn.outlier_elements(shape, 7), "grid": lambda: syn.grid_values(shape, 8)}[kind]()
    x = syn.bf16_bits_to_f32(bits)
    s_T = F32(qn.nvfp4_tensor_scale(qn.abs_max(x), qn.NV_RTN_DIV) * F32(scale_factor))
    _check(x, s_T)


def test_kernel_search_order_on_extreme_scales_and_sparse_groups():
    rng = np.random.default_rng(51)
    x = rng.standard_normal((64, 16)).astype(F32)
    x[::3] = 0.0
    x[1::3, 1:] = 0.0                                         # one non-zero value per group
    for s_T in (F32(1e-38), F32(3e-41), F32(1e30), F32(2e36), F32(1.0)):
        _check((x * F32(1e-36)).astype(F32), s_T)
        _check((x * F32(1e37)).astype(F32), s_T)
        _check(x, s_T)
