"""Parity at the benchmarked sizes, on sampled outputs.

The quantisers, the GEMM and the linear layer run on the GPU at the full
sizes of the workloads (the Llama-3-8B-shaped layer set at M = 16384, the
Quartet II layer 8192 x 2048 -> 8192, the Quartet layer 4096 x 2048 -> 2048,
a 2^28-element quantiser-sweep tensor), in the launch configuration bench.py
times.  The oracle recomputes a sample of output rows from the same bf16
inputs: rotation, scales and codes are row-local, the NVFP4 tensor scale
needs the whole transformed tensor's max |y| (computed by the oracle in row
chunks) and the stochastic modes index Philox by the rows' positions in the
whole tensor (``oracle.quant.quantize_rows``, pinned against the whole-tensor
quantiser on CPU).  GEMM outputs are checked on sampled rows x columns
against fp64 dot products of the oracle's own quantised rows; nothing the
GPU computed is fed to the oracle."""
import numpy as np
import pytest
import torch

from fp4_microscaled_quantized_b200 import synthetic as syn
from oracle import formats as fm
from oracle import gemm as gm
from oracle import linear as ln
from oracle import quant as qn

pytestmark = pytest.mark.gpu


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def f32(bits):
    return syn.bf16_bits_to_f32(bits)


def sample(n, k=16, seed=0, align=1):
    """First k, last k and k random indices in [0, n) (multiples of `align`
    when a block of `align` consecutive indices is wanted)."""
    nb = n // align
    r = np.random.default_rng(seed)
    idx = np.unique(np.concatenate([np.arange(min(k, nb)), np.arange(max(nb - k, 0), nb),
                                    r.integers(0, nb, k)]))
    return idx if align == 1 else (idx[:, None] * align + np.arange(align)[None, :]).ravel()


def swz_offsets(rows, ngroups, total_rows):
    """Byte offsets of (row, group) in the tensor-core scale layout."""
    nkb = (ngroups + 3) // 4
    r = rows[:, None].astype(np.int64)
    k = np.arange(ngroups, dtype=np.int64)[None, :]
    return ((r // 128) * nkb + k // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + k % 4


def check_rows(g, o, rows):
    """GPU QTensor rows `rows` equal the oracle's sampled QTensor bit for bit."""
    torch.cuda.synchronize()
    ri = torch.from_numpy(rows).cuda()
    np.testing.assert_array_equal(g.codes.index_select(0, ri).cpu().numpy(), fm.pack_codes(o.codes))
    np.testing.assert_array_equal(g.scales.index_select(0, ri).cpu().numpy(), o.scales)
    off = swz_offsets(rows, o.scales.shape[1], g.codes.shape[0])
    swz = g.scales_swz.cpu().numpy()
    np.testing.assert_array_equal(swz[off], o.scales)
    assert g.tensor_scale.item() == float(o.tensor_scale)
    if o.mask is not None:
        np.testing.assert_array_equal(g.mask.index_select(0, ri).cpu().numpy(), fm.pack_mask(o.mask))


def check_block(y, rows, cols, y_ref, bound):
    torch.cuda.synchronize()
    got = y.index_select(0, torch.from_numpy(rows).cuda()).index_select(
        1, torch.from_numpy(cols).cuda()).float().cpu().numpy().astype(np.float64)
    err = np.abs(got - y_ref)
    assert np.all(err <= bound), "max excess %g" % (err - bound).max()


# ------------------------------------------------------------ quantisers --
QCASES = {
    # the backward operands of the QKV layer at M = 16384 (dY 16384 x 6144, Student-t x 1e-3)
    "E_row_ms_eden": ("dy", qn.NVFP4, qn.MS_EDEN, 128, False, ln.GEMM_DX, ln.TAG_E_ROW),
    "E_t_ms_eden": ("dy", qn.NVFP4, qn.MS_EDEN, 128, True, ln.GEMM_DW, ln.TAG_E_T),
    # its forward operands (X 16384 x 4096 Student-t at unit RMS, W 6144 x 4096)
    "X_four_over_six": ("x", qn.NVFP4, qn.FOUR_OVER_SIX, 0, False, 0, ln.TAG_X),
    "W_four_over_six": ("w", qn.NVFP4, qn.FOUR_OVER_SIX, 0, False, 0, ln.TAG_W),
    # the quantiser sweep's 2^28-element point (rows of 4096, N(0,1) + 0.1% x 50)
    "sweep_2e28_nvfp4_sr_h32": ("sweep", qn.NVFP4, qn.SR, 32, False, 0, 9),
    "sweep_2e28_nvfp4_eden_h128_t": ("sweep", qn.NVFP4, qn.MS_EDEN, 128, True, 1, 10),
    "sweep_2e28_nvfp4_fos_h0": ("sweep", qn.NVFP4, qn.FOUR_OVER_SIX, 0, False, 0, 11),
    "sweep_2e28_mxfp4_quest_h32": ("sweep", qn.MXFP4, qn.QUEST, 32, False, 0, 12),
}


@pytest.fixture(scope="module")
def qkv_data():
    return syn.linear_quartet2(16384, 6144, 4096, seed=3)


@pytest.fixture(scope="module")
def sweep_data():
    return syn.quantizer_sweep(1 << 28)


@pytest.mark.parametrize("name", list(QCASES))
def test_quantizer_full_size(cuda_lib, qkv_data, request, name):
    src, fmt, rnd, had, transpose, sign_tag, tag = QCASES[name]
    bits = request.getfixturevalue("sweep_data") if src == "sweep" else \
        {"dy": qkv_data["dY"], "x": qkv_data["X"], "w": qkv_data["W"]}[src]
    seed = 1234
    rand = had > 0 and rnd in (qn.SR, qn.MS_EDEN)      # the backward modes rotate randomly, the others do not
    g = cuda_lib.quantize(dev(bits), fmt, rnd, had, randomized=rand, seed=seed, sign_tag=sign_tag,
                          tensor_tag=tag, transpose=transpose)
    n_out = bits.shape[1] if transpose else bits.shape[0]
    rows = sample(n_out, seed=len(name))
    o = qn.quantize_rows(f32(bits), rows, fmt, rnd, had, randomized=rand, seed=seed, sign_tag=sign_tag,
                         tensor_tag=tag, transpose=transpose)
    check_rows(g, o, rows)
    assert cuda_lib.get_last_error() == 0


def test_requantize_full_size(cuda_lib, qkv_data):
    """Saved Q(W) of the QKV layer -> dequantise -> transpose -> RHT128 ->
    MS-EDEN (the dX operand), from the oracle's own Q(W)."""
    W = qkv_data["W"]
    gq = cuda_lib.quantize(dev(W), qn.NVFP4, qn.FOUR_OVER_SIX)
    g = cuda_lib.requantize(gq, qn.MS_EDEN, 128, randomized=True, seed=77, sign_tag=ln.GEMM_DX,
                            tensor_tag=ln.TAG_W_T, transpose=True)
    oq = qn.nvfp4_four_over_six(f32(W))
    deq = qn.dequant_f32(oq)
    rows = sample(W.shape[1], seed=5)
    o = qn.quantize_rows(deq, rows, qn.NVFP4, qn.MS_EDEN, 128, randomized=True, seed=77,
                         sign_tag=ln.GEMM_DX, tensor_tag=ln.TAG_W_T, transpose=True)
    check_rows(g, o, rows)
    assert cuda_lib.get_last_error() == 0


# ------------------------------------------------------------------ GEMM --
@pytest.mark.parametrize("layer", [l[0] for l in syn.LLAMA3_8B_LAYERS])
def test_gemm_full_size_layer_forward(cuda_lib, layer):
    """Y = Q(X) Q(W)^T of each Llama-3-8B-shaped layer at M = 16384 (the
    CTA-pair kernel), 48 x 48 sampled outputs."""
    i = [l[0] for l in syn.LLAMA3_8B_LAYERS].index(layer)
    _, K, N = syn.LLAMA3_8B_LAYERS[i]
    # X and W of syn.linear_quartet2(16384, N, K, seed=3 + i), without its dY
    d = {"X": syn.student_t((16384, K), 3 + i, 0, unit_rms=True), "W": syn.gaussian((N, K), 0.02, 3 + i, 1)}
    A = cuda_lib.quantize(dev(d["X"]), qn.NVFP4, qn.FOUR_OVER_SIX)
    B = cuda_lib.quantize(dev(d["W"]), qn.NVFP4, qn.FOUR_OVER_SIX)
    Y = cuda_lib.gemm(A, B)
    rows, cols = sample(16384, seed=i), sample(N, seed=10 + i)
    oa = qn.quantize_rows(f32(d["X"]), rows, qn.NVFP4, qn.FOUR_OVER_SIX)
    ob = qn.quantize_rows(f32(d["W"]), cols, qn.NVFP4, qn.FOUR_OVER_SIX)
    y_ref, bound = gm.gemm_ref(oa, ob)
    check_block(Y, rows, cols, y_ref, bound)
    assert cuda_lib.get_last_error() == 0


# ---------------------------------------------------------- linear layer --
def test_linear_quartet2_full_size(cuda_lib):
    """Quartet II layer M = 8192, K = 2048, N = 8192 through fp4_linear_fwd /
    fp4_linear_bwd: the saved context on sampled rows, Y, dX and dW on
    sampled rows x columns."""
    M, N, K, step = 8192, 8192, 2048, 11
    d = syn.linear_quartet2(M, N, K, seed=2)
    X, W, dY = f32(d["X"]), f32(d["W"]), f32(d["dY"])
    r = cuda_lib.recipe(cuda_lib.RECIPE_QUARTET2)
    Y, ctx = cuda_lib.linear_fwd(dev(d["X"]), dev(d["W"]), r, seed=0)
    dX, dW = cuda_lib.linear_bwd(dev(d["dY"]), ctx, step)
    rm, rn, rk = sample(M, seed=1), sample(N, seed=2), sample(K, seed=3)
    oxq = qn.quantize_rows(X, rm, qn.NVFP4, qn.FOUR_OVER_SIX)
    owq = qn.quantize_rows(W, rn, qn.NVFP4, qn.FOUR_OVER_SIX)
    check_rows(ctx.xq, oxq, rm)
    check_rows(ctx.wq, owq, rn)
    y_ref, yb = gm.gemm_ref(oxq, owq)
    check_block(Y, rm, rn, y_ref, yb)
    # backward operands from the oracle's own saved Q(X), Q(W)
    deq_x = qn.dequant_f32(qn.nvfp4_four_over_six(X))
    deq_w = qn.dequant_f32(qn.nvfp4_four_over_six(W))
    kw = dict(randomized=True, seed=step)
    e_row = qn.quantize_rows(dY, rm, qn.NVFP4, qn.MS_EDEN, 128, sign_tag=ln.GEMM_DX, tensor_tag=ln.TAG_E_ROW, **kw)
    w_t = qn.quantize_rows(deq_w, rk, qn.NVFP4, qn.MS_EDEN, 128, sign_tag=ln.GEMM_DX, tensor_tag=ln.TAG_W_T,
                           transpose=True, **kw)
    dx_ref, dxb = gm.gemm_ref(e_row, w_t)
    check_block(dX, rm, rk, dx_ref, dxb)
    e_t = qn.quantize_rows(dY, rn, qn.NVFP4, qn.MS_EDEN, 128, sign_tag=ln.GEMM_DW, tensor_tag=ln.TAG_E_T,
                           transpose=True, **kw)
    x_t = qn.quantize_rows(deq_x, rk, qn.NVFP4, qn.MS_EDEN, 128, sign_tag=ln.GEMM_DW, tensor_tag=ln.TAG_X_T,
                           transpose=True, **kw)
    dw_ref, dwb = gm.gemm_ref(e_t, x_t)
    check_block(dW, rn, rk, dw_ref, dwb)
    assert cuda_lib.get_last_error() == 0


def test_linear_quartet_full_size(cuda_lib):
    """Quartet (MXFP4) layer M = 4096, K = N = 2048: QuEST + H32 forward with
    clip masks, SR(3/4 RHT32) backward and the 16/9 H32^-1 mask epilogue,
    sampled rows x aligned 32-column blocks."""
    M, N, K, step = 4096, 2048, 2048, 21
    d = syn.linear_quartet(M, N, K, seed=1)
    X, W, dY = f32(d["X"]), f32(d["W"]), f32(d["dY"])
    r = cuda_lib.recipe(cuda_lib.RECIPE_QUARTET)
    Y, ctx = cuda_lib.linear_fwd(dev(d["X"]), dev(d["W"]), r, seed=0)
    dX, dW = cuda_lib.linear_bwd(dev(d["dY"]), ctx, step)
    rec = ln.QUARTET
    rm, rn = sample(M, k=8, seed=1), sample(N, k=8, seed=2)
    kb = sample(K, k=2, seed=3, align=32)              # whole 32-column blocks (the inverse H32)
    nb = sample(N, k=2, seed=4, align=32)
    oxq = qn.quantize_rows(X, rm, rec.fmt, rec.fwd_rnd, rec.fwd_had, tensor_tag=ln.TAG_X)
    owq = qn.quantize_rows(W, rn, rec.fmt, rec.fwd_rnd, rec.fwd_had, tensor_tag=ln.TAG_W)
    check_rows(ctx.xq, oxq, rm)
    check_rows(ctx.wq, owq, rn)
    y_ref, yb = gm.gemm_ref(oxq, owq)
    check_block(Y, rm, rn, y_ref, yb)
    kw = dict(randomized=True, seed=step)
    deq_x = qn.dequant_f32(qn.quantize(X, rec.fmt, rec.fwd_rnd, rec.fwd_had, tensor_tag=ln.TAG_X))
    deq_w = qn.dequant_f32(qn.quantize(W, rec.fmt, rec.fwd_rnd, rec.fwd_had, tensor_tag=ln.TAG_W))
    mask_x = qn.quantize_rows(X, rm, rec.fmt, rec.fwd_rnd, rec.fwd_had).mask[:, kb]
    mask_w = qn.quantize_rows(W, nb, rec.fmt, rec.fwd_rnd, rec.fwd_had).mask[:, kb]
    e_row = qn.quantize_rows(dY, rm, rec.fmt, rec.bwd_rnd, rec.bwd_had, sign_tag=ln.GEMM_DX,
                             tensor_tag=ln.TAG_E_ROW, **kw)
    w_t = qn.quantize_rows(deq_w, kb, rec.fmt, rec.bwd_rnd, rec.bwd_had, sign_tag=ln.GEMM_DX,
                           tensor_tag=ln.TAG_W_T, transpose=True, **kw)
    dx, bx = gm.gemm_ref(e_row, w_t)
    dx_ref, dxb = gm.quartet_epilogue_ref(dx, bx, ~mask_x, rec.fwd_had)
    check_block(dX, rm, kb, dx_ref, dxb)
    e_t = qn.quantize_rows(dY, nb, rec.fmt, rec.bwd_rnd, rec.bwd_had, sign_tag=ln.GEMM_DW,
                           tensor_tag=ln.TAG_E_T, transpose=True, **kw)
    x_t = qn.quantize_rows(deq_x, kb, rec.fmt, rec.bwd_rnd, rec.bwd_had, sign_tag=ln.GEMM_DW,
                           tensor_tag=ln.TAG_X_T, transpose=True, **kw)
    dw, bw = gm.gemm_ref(e_t, x_t)
    dw_ref, dwb = gm.quartet_epilogue_ref(dw, bw, ~mask_w, rec.fwd_had)
    check_block(dW, nb, kb, dw_ref, dwb)
    assert cuda_lib.get_last_error() == 0


def test_linear_layer_set_gate_up_full_size(cuda_lib):
    """The layer set's gate/up layer at M = 16384 (K = 4096, N = 28672, data
    seed 5 as in the bench) through fp4_linear_fwd / fp4_linear_bwd: the two
    longest accumulations the bench times, dX = E W (inner N = 28672) and
    dW = E^T X (inner M = 16384), on sampled rows x columns against fp64
    products of the oracle's own operands (its whole-tensor Four-Over-Six of
    X and W, de-quantised, and its MS-EDEN of the sampled rows with the
    whole transformed tensors' amax)."""
    M, K, N, step = 16384, 4096, 28672, 3
    d = syn.linear_quartet2(M, N, K, seed=5)
    r = cuda_lib.recipe(cuda_lib.RECIPE_QUARTET2)
    Y, ctx = cuda_lib.linear_fwd(dev(d["X"]), dev(d["W"]), r, seed=0)
    dX, dW = cuda_lib.linear_bwd(dev(d["dY"]), ctx, step)
    torch.cuda.synchronize()
    X, W, dY = f32(d["X"]), f32(d["W"]), f32(d["dY"])
    del d
    rm, rn, rk = sample(M, k=12, seed=31), sample(N, k=12, seed=32), sample(K, k=12, seed=33)
    oxq, owq = qn.nvfp4_four_over_six(X), qn.nvfp4_four_over_six(W)
    check_rows(ctx.xq, qn.QTensor(oxq.codes[rm], oxq.scales[rm], oxq.tensor_scale, oxq.fmt), rm)
    y_ref, yb = gm.gemm_ref(qn.QTensor(oxq.codes[rm], oxq.scales[rm], oxq.tensor_scale, oxq.fmt),
                            qn.QTensor(owq.codes[rn], owq.scales[rn], owq.tensor_scale, owq.fmt))
    check_block(Y, rm, rn, y_ref, yb)
    deq_x, deq_w = qn.dequant_f32(oxq), qn.dequant_f32(owq)
    del oxq, owq, X, W
    kw = dict(randomized=True, seed=step)
    e_row = qn.quantize_rows(dY, rm, qn.NVFP4, qn.MS_EDEN, 128, sign_tag=ln.GEMM_DX, tensor_tag=ln.TAG_E_ROW, **kw)
    w_t = qn.quantize_rows(deq_w, rk, qn.NVFP4, qn.MS_EDEN, 128, sign_tag=ln.GEMM_DX, tensor_tag=ln.TAG_W_T,
                           transpose=True, **kw)
    dx_ref, dxb = gm.gemm_ref(e_row, w_t)
    check_block(dX, rm, rk, dx_ref, dxb)
    e_t = qn.quantize_rows(dY, rn, qn.NVFP4, qn.MS_EDEN, 128, sign_tag=ln.GEMM_DW, tensor_tag=ln.TAG_E_T,
                           transpose=True, **kw)
    x_t = qn.quantize_rows(deq_x, rk, qn.NVFP4, qn.MS_EDEN, 128, sign_tag=ln.GEMM_DW, tensor_tag=ln.TAG_X_T,
                           transpose=True, **kw)
    dw_ref, dwb = gm.gemm_ref(e_t, x_t)
    check_block(dW, rn, rk, dw_ref, dwb)
    assert cuda_lib.get_last_error() == 0
