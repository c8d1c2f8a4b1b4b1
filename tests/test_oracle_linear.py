"""Pins of the oracle GEMM reference and linear-layer recipes."""
import numpy as np
import pytest

from fp4_microscaled_quantized_b200 import synthetic as syn
from oracle import gemm as gm
from oracle import hadamard as hd
from oracle import linear as ln
from oracle import quant as qn

F32 = np.float32


def _cos(a, b):
    a, b = a.reshape(-1), b.reshape(-1)
    return float(a @ b / np.linalg.norm(a) / np.linalg.norm(b))


def test_gemm_ref_brute_force():
    rng = np.random.default_rng(0)
    A = qn.nvfp4_rtn(rng.standard_normal((5, 32)).astype(F32))
    B = qn.nvfp4_four_over_six(rng.standard_normal((3, 32)).astype(F32))
    y, b = gm.gemm_ref(A, B)
    a64, b64 = qn.dequant_f64(A), qn.dequant_f64(B)
    for i in range(5):
        for j in range(3):
            s = sum(a64[i, k] * b64[j, k] for k in range(32))
            assert abs(y[i, j] - s) <= 1e-12 * max(1.0, abs(s))
            assert b[i, j] > 0
    yi, bi = gm.gemm_ref_sampled(A, B, np.array([4, 0, 2]), np.array([1, 2, 0]))
    np.testing.assert_allclose(yi, [y[4, 1], y[0, 2], y[2, 0]], rtol=1e-12)


def test_lossless_gemm_is_exact():
    """Grid values with power-of-two scales quantise losslessly, so the
    reference equals the exact product."""
    rng = np.random.default_rng(1)
    ca = rng.integers(0, 16, (16, 64)).astype(np.uint8); ca[:, ::32] = 7
    cb = rng.integers(0, 16, (8, 64)).astype(np.uint8); cb[:, ::32] = 7
    from oracle import formats as fm
    a = fm.decode_e2m1(ca).astype(np.float64) * 2.0 ** -3
    b = fm.decode_e2m1(cb).astype(np.float64) * 2.0 ** 2
    y, _ = gm.gemm_ref(qn.mxfp4_rtn(a.astype(F32)), qn.mxfp4_rtn(b.astype(F32)))
    np.testing.assert_array_equal(y, a @ b.T)


def _layer(M, N, K, seed):
    d = syn.linear_quartet(M, N, K, seed)
    return {k: syn.bf16_bits_to_f32(v) for k, v in d.items()}


def test_quartet_forward_and_backward_track_exact_gradients():
    M, N, K = 256, 128, 256
    t = _layer(M, N, K, 3)
    X, W, dY = t["X"], t["W"], t["dY"]
    y, b, ctx = ln.linear_fwd(X, W, ln.QUARTET)
    exact = X.astype(np.float64) @ W.astype(np.float64).T
    assert _cos(y, exact) > 0.98
    (dx, bx), (dw, bw), ops = ln.linear_bwd(dY, ctx, ln.QUARTET, step_seed=7)
    assert dx.shape == (M, K) and dw.shape == (N, K)
    # straight-through reference: zero the gradient at clipped elements in the
    # Hadamard domain, then transform back
    dxh = dY.astype(np.float64) @ hd.block_transform_f64(W, 32, False)
    dx_ste = hd.inverse_block_h_f64(dxh * ~ctx["Xq"].mask, 32)
    dwh = dY.astype(np.float64).T @ hd.block_transform_f64(X, 32, False)
    dw_ste = hd.inverse_block_h_f64(dwh * ~ctx["Wq"].mask, 32)
    assert _cos(dx, dx_ste) > 0.9 and _cos(dw, dw_ste) > 0.9
    # a transposed operand or a missing inverse transform is far off
    assert _cos(dx, dxh * ~ctx["Xq"].mask) < 0.5
    # the 16/9 is carried by the two 4/3 tensor scales
    assert float(ops["E_row"].tensor_scale) * float(ops["W_t"].tensor_scale) == np.float32(4 / 3) ** 2


@pytest.mark.parametrize("recipe", [ln.QUARTET2, ln.TETRAJET2, ln.NVIDIA], ids=["quartet2", "tetrajet2", "nvidia"])
def test_quartet2_backward_is_unbiased_in_the_mean(recipe):
    M, N, K = 128, 128, 256
    d = syn.linear_quartet2(M, N, K, 4)
    X, W, dY = (syn.bf16_bits_to_f32(d[k]) for k in ("X", "W", "dY"))
    _, _, ctx = ln.linear_fwd(X, W, recipe)
    # target: the product with the saved (forward-quantised) operands
    wq = qn.dequant_f64(ctx["Wq"])
    xq = qn.dequant_f64(ctx["Xq"])
    tgt_dx = dY.astype(np.float64) @ wq
    tgt_dw = dY.astype(np.float64).T @ xq
    acc_dx = np.zeros_like(tgt_dx)
    acc_dw = np.zeros_like(tgt_dw)
    n = 16
    single = None
    for s in range(n):
        (dx, _), (dw, _), _ = ln.linear_bwd(dY, ctx, recipe, step_seed=s)
        acc_dx += dx
        acc_dw += dw
        if single is None:
            single = np.linalg.norm(dx - tgt_dx)
    err_mean = np.linalg.norm(acc_dx / n - tgt_dx)
    assert err_mean < 0.5 * single                       # about 1/sqrt(16)
    assert _cos(acc_dw / n, tgt_dw) > 0.99


def test_rtn_recipe_forward():
    d = syn.linear_rtn_small(0)
    X, W = syn.bf16_bits_to_f32(d["X"]), syn.bf16_bits_to_f32(d["W"])
    y, b, ctx = ln.linear_fwd(X, W, ln.RTN)
    assert y.shape == (256, 512)
    assert _cos(y, X.astype(np.float64) @ W.astype(np.float64).T) > 0.98
    assert ctx["Xq"].mask is None


def test_epilogue_bound_propagation():
    rng = np.random.default_rng(5)
    y = rng.standard_normal((4, 64))
    bound = np.abs(rng.standard_normal((4, 64))) * 1e-3
    keep = rng.random((4, 64)) > 0.1
    out, ob = gm.quartet_epilogue_ref(y, bound, keep)
    ref = hd.inverse_block_h_f64(y * keep, 32)
    np.testing.assert_allclose(out, ref)
    h = np.abs(hd.sylvester(32)) / np.sqrt(32)
    for r in range(4):
        for blk in range(2):
            sl = slice(32 * blk, 32 * blk + 32)
            np.testing.assert_allclose(ob[r, sl], h @ (bound[r, sl] * keep[r, sl]))


def test_ms_eden_backward_beats_sr_backward():
    """The Quartet II page's comparison with the simplified TetraJet-v2: the
    same backward graph with MS-EDEN in place of SR estimates both gradients
    with less error (per-tensor MSE more than 2x lower, "Table 1"; Figure 1)."""
    M, N, K = 256, 256, 512
    d = syn.linear_quartet2(M, N, K, 6)
    X, W, dY = (syn.bf16_bits_to_f32(d[k]) for k in ("X", "W", "dY"))
    err = {}
    for name, r in (("eden", ln.QUARTET2), ("sr", ln.TETRAJET2)):
        _, _, ctx = ln.linear_fwd(X, W, r)
        tgt_dx = dY.astype(np.float64) @ qn.dequant_f64(ctx["Wq"])
        tgt_dw = dY.astype(np.float64).T @ qn.dequant_f64(ctx["Xq"])
        e = [0.0, 0.0]
        for s in range(4):
            (dx, _), (dw, _), _ = ln.linear_bwd(dY, ctx, r, step_seed=s)
            e[0] += np.sum((dx - tgt_dx) ** 2)
            e[1] += np.sum((dw - tgt_dw) ** 2)
        err[name] = e
    assert err["eden"][0] < 0.7 * err["sr"][0]
    assert err["eden"][1] < 0.7 * err["sr"][1]


def test_nvidia_recipe_reuses_the_forward_weights():
    """The NVIDIA recipe's dX GEMM multiplies by the forward Q(W) itself
    (square blocks, transposed), so with SR on dY the mean over seeds
    converges to dY Q(W) and the re-used operand equals Q(W^T) quantised
    directly from W^T."""
    M, N, K = 128, 128, 256
    d = syn.linear_quartet2(M, N, K, 8)
    X, W, dY = (syn.bf16_bits_to_f32(d[k]) for k in ("X", "W", "dY"))
    _, _, ctx = ln.linear_fwd(X, W, ln.NVIDIA)
    ops = ln.bwd_operands(dY, ctx, ln.NVIDIA, 3)
    direct = qn.quantize(W, qn.NVFP4, qn.RTN_SQUARE16, 0, transpose=True)
    np.testing.assert_array_equal(ops["W_t"].codes, direct.codes)
    np.testing.assert_array_equal(ops["W_t"].scales, direct.scales)
