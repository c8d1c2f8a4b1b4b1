"""Method diagnostics on synthetic data, computed with the library's kernels.

* Quantisation MSE on N(0, 1) vectors for every format and rounding mode --
  the Quartet II page's Table 1 ("Practical Performance of MS-EDEN": NVFP4
  SR 23.5, MS-EDEN 9.8, RTN 9.0, RTN + 4/6 7.6, RTN with 16 x 16 scales 12.4,
  all x 1e-3) and the MXFP4
  error column of the Quartet page's Table 2.
* Projection magnitude misalignment 1 - E[1/S], S = <X, X> / <H(X), Q(H(X))>,
  over random rotations H (Quartet page, "Backward-Pass Quantization"): zero
  for an unbiased quantiser (the page prints 0.00 for SR), non-zero for RTN.
* Unbiasedness in the mean (Quartet II page, "Unbiasedness Verification",
  Figure 9): the mean of B de-quantised, back-rotated samples over independent
  rotation / rounding seeds approaches the input with an error falling like
  1/B for an unbiased quantiser (MS-EDEN, SR), and levels off for RTN.

Quantisation, rotation and de-quantisation run in the CUDA library through
its C ABI; only the final reductions (mean square, inner products) and the
back-rotation of the de-quantised samples use torch.
"""
import numpy as np
import torch

from . import api
from . import synthetic as syn

# Table 1 of the Quartet II page (NVFP4, native 1x16 scales, MSE x 1e-3).
TABLE1_NVFP4 = {"rtn": 9.0, "fos": 7.6, "sr": 23.5, "eden": 9.8, "rtn16x16": 12.4}

NAMES = {api.RTN: "rtn", api.QUEST: "quest", api.FOUR_OVER_SIX: "fos", api.SR: "sr", api.MS_EDEN: "eden",
         api.RTN_SQUARE16: "rtn16x16"}


def _dev(bits, device):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def roundtrip(x, fmt, rnd, had, seed=0, sign_tag=0):
    """(rotated input y, de-quantised Q(y)) as fp32 device tensors for a bf16
    device tensor x: y = H_had(x) (randomized for SR and MS-EDEN, x itself
    without a rotation), Q the quantiser (format, rounding) applied to it."""
    rand = rnd in (api.SR, api.MS_EDEN) and had > 0
    q = api.quantize(x, fmt, rnd, had, randomized=rand, seed=seed, sign_tag=sign_tag, tensor_tag=1)
    dq = api.dequantize(q)
    y = api.hadamard(x, had, randomized=rand, seed=seed, sign_tag=sign_tag) if had else x.float()
    return y, dq


def quant_mse(fmt, rnd, had, rows=1024, cols=1024, seed=0, n_seeds=2, device="cuda"):
    """Mean squared quantisation error x 1e3 of N(0, 1) data (2^20 values by
    default), in the rotated domain (the rotation is orthonormal), averaged
    over `n_seeds` rotation / rounding seeds for the random modes."""
    x = _dev(syn.gaussian((rows, cols), 1.0, seed), device)
    seeds = range(n_seeds) if (rnd in (api.SR, api.MS_EDEN)) else range(1)
    acc = 0.0
    for s in seeds:
        y, dq = roundtrip(x, fmt, rnd, had, seed=s)
        acc += float(torch.mean((dq.double() - y.double()) ** 2))
    return 1e3 * acc / len(seeds)


def misalignment(fmt, rnd, had, rows=256, cols=4096, n_seeds=64, seed=3, device="cuda"):
    """1 - E[1/S] with 1/S = <H(X), Q(H(X))> / <X, X> per row vector X
    (gradient-like: 1e-3 x Student-t(3) values), averaged over `n_seeds`
    random rotations; returns (value, standard error over rows x seeds)."""
    bits = syn.student_t((rows, cols), seed, scale=1e-3)
    x = _dev(bits, device)
    xx = (x.double() ** 2).sum(dim=1)
    inv_s = []
    for s in range(n_seeds):
        y, dq = roundtrip(x, fmt, rnd, had, seed=1000 + s)
        inv_s.append(((y.double() * dq.double()).sum(dim=1) / xx).cpu())
    v = torch.stack(inv_s).flatten()
    return float(1.0 - v.mean()), float(v.std() / np.sqrt(v.numel()))


def mean_convergence(fmt, rnd, had, n=10000, cols=1024, seed=14, Bs=(10, 100, 1000, 10000), device="cuda"):
    """Relative squared error |mean_B - x|^2 / |x|^2 of the mean of the first B
    of n samples RHT_s^-1(Q(RHT_s(x))), s = 0 .. n-1, for each B in `Bs`, and
    the log-log slope over Bs (-1 for an unbiased quantiser).  x: 1 x cols of
    N(0,1).  The back-rotation of seed s is the transpose of the matrix whose
    rows are the rotated unit vectors (fp4_hadamard of the identity)."""
    x = _dev(syn.gaussian((1, cols), 1.0, seed), device)
    xd = x.double().view(-1)
    eye = torch.eye(had, dtype=torch.bfloat16, device=device)
    acc = torch.zeros((n, cols), dtype=torch.float64, device=device)
    for s in range(n):
        q = api.quantize(x, fmt, rnd, had, randomized=True, seed=s, sign_tag=0, tensor_tag=1)
        dq = api.dequantize(q).double()
        rot = api.hadamard(eye, had, randomized=True, seed=s, sign_tag=0).double()
        acc[s] = (dq.view(-1, had) @ rot.T).view(-1)
    Bs = [b for b in Bs if b <= n]
    errs = [float(((acc[:b].mean(0) - xd) ** 2).sum() / (xd ** 2).sum()) for b in Bs]
    slope = float(np.polyfit(np.log(Bs), np.log(errs), 1)[0])
    rel_bias = float((acc.mean(0) - xd).norm() / xd.norm())
    return {"B": Bs, "rel_sq_err": errs, "slope": slope, "rel_bias": rel_bias}


def table(device="cuda"):
    """Every (format, rounding, rotation) the diagnostics cover, as dicts."""
    out = []
    for rnd, had in ((api.RTN, 0), (api.FOUR_OVER_SIX, 0), (api.SR, 0), (api.MS_EDEN, 128), (api.RTN_SQUARE16, 0)):
        out.append({"format": "nvfp4", "rounding": NAMES[rnd], "had": had,
                    "mse_x1e3": quant_mse(api.NVFP4, rnd, had, device=device),
                    "page_mse_x1e3": TABLE1_NVFP4[NAMES[rnd]]})
    for rnd in (api.RTN, api.QUEST, api.SR):
        out.append({"format": "mxfp4", "rounding": NAMES[rnd], "had": 32,
                    "mse_x1e3": quant_mse(api.MXFP4, rnd, 32, device=device)})
    for fmt, rnd, had in ((api.MXFP4, api.SR, 32), (api.MXFP4, api.RTN, 32), (api.MXFP4, api.QUEST, 32),
                          (api.NVFP4, api.SR, 128), (api.NVFP4, api.MS_EDEN, 128), (api.NVFP4, api.RTN, 128)):
        m, se = misalignment(fmt, rnd, had, device=device)
        out.append({"format": "mxfp4" if fmt == api.MXFP4 else "nvfp4", "rounding": NAMES[rnd], "had": had,
                    "misalignment": m, "misalignment_stderr": se})
    for fmt, rnd, had in ((api.NVFP4, api.MS_EDEN, 128), (api.NVFP4, api.SR, 128), (api.NVFP4, api.RTN, 128)):
        r = mean_convergence(fmt, rnd, had, device=device)
        out.append({"format": "nvfp4", "rounding": NAMES[rnd], "had": had, "mean_convergence": r})
    return out
