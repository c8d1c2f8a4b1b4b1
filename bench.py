#!/usr/bin/env python
"""Benchmark of the fully-FP4 linear layer on B200.

Workloads (``--config``):
  4 (default) the Llama-3-8B-shaped layer set in the Quartet II NVFP4 recipe,
    M = 16384 tokens, layers QKV 4096->6144, O 4096->4096, gate/up
    4096->28672 (2 x 14336 as one GEMM), down 14336->4096;
  3 one Quartet II NVFP4 layer, M = 8192, K = 2048, N = 8192;
  2 one Quartet MXFP4 layer, M = 4096, K = N = 2048 (QuEST + H32 forward, SR
    of the RHT-32 backward, the mask / inverse-Hadamard epilogue);
  1 a single NVFP4 RTN forward linear, X 256x512, W 512x512 (latency).
One step = forward + backward of every layer (forward only for config 1)
through the C ABI's fp4_linear_fwd / fp4_linear_bwd.  Metric: TFLOP/s =
6 M sum(N K) / step time (2 M N K for config 1, reported as latency too).

  python bench.py [--config C] [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

The JSON line's `value` is timed through the linear entry points alone.  A
second timed region of the same length issues the same kernels through the
primitive entry points with CUDA events around each call, for the per-kernel
split and the roofline figures.  N > 1 runs N independent replicas (one per
rank, launched by torchrun); the step time is the max over ranks.  Prints one
JSON line on rank 0.
"""
import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

# The oracle's all-core timing runs in spawned worker processes, which import
# this file as "__mp_main__"; they run numpy code only and skip torch.
if __name__ != "__mp_main__":
    import torch  # noqa: E402

from fp4_microscaled_quantized_b200 import synthetic as syn  # noqa: E402

METRIC = "NVFP4 linear fwd+bwd TFLOPS and quantizer HBM GB/s vs roofline, 1xB200"
UNIT = "TFLOP/s"
M_TOKENS = 16384
LAYERS = syn.LLAMA3_8B_LAYERS          # (name, K = in_features, N = out_features)
TAG_E_ROW, TAG_W_T, TAG_E_T, TAG_X_T, TAG_X, TAG_W = 1, 2, 3, 4, 5, 6
GEMM_DX, GEMM_DW = 0, 1
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_OVER_BF16 = 4.0                    # nominal dense ratio 9 / 2.25 PFLOP/s
SUSTAINED_AFTER_S = 2.0                # timed regions at least this long use the sustained peak
L2_FLUSH_BYTES = 256 << 20             # larger than the 126 MB L2

# Workloads: (name, M, layers (name, K, N), recipe preset name, backward?, data)
CONFIGS = {
    1: {"workload": "single NVFP4 RTN forward linear, X 256x512 ~N(0,1), W 512x512 ~N(0,0.02^2), "
                    "no Hadamard, seed 0",
        "M": 256, "layers": (("linear", 512, 512),), "recipe": "rtn", "bwd": False, "flush": True, "seed": 0},
    2: {"workload": "Quartet MXFP4 linear fwd+bwd, M=4096, K=N=2048 (QuEST+H32 fwd, SR of RHT32 bwd, "
                    "mask/H32^-1 epilogue)",
        "M": 4096, "layers": (("linear", 2048, 2048),), "recipe": "quartet", "bwd": True, "flush": True, "seed": 1},
    3: {"workload": "Quartet II NVFP4 linear fwd+bwd, M=8192, K=2048, N=8192 (4/6 fwd, RHT128 + MS-EDEN bwd)",
        "M": 8192, "layers": (("linear", 2048, 8192),), "recipe": "quartet2", "bwd": True, "flush": True,
        "seed": 2},
    4: {"workload": "llama3-8b layer set (qkv 4096->6144, o 4096->4096, gate_up 4096->28672, "
                    "down 14336->4096), NVFP4 Quartet II fwd+bwd",
        "M": M_TOKENS, "layers": LAYERS, "recipe": "quartet2", "bwd": True, "flush": False, "seed": 3},
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", type=int, choices=sorted(CONFIGS), default=4)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=None, help="override M (profiling small cases)")
    ap.add_argument("--layers", default="qkv,o,gate_up,down",
                    help="subset of config 4's layer set (profiling small cases)")
    ap.add_argument("--quant-sweep", action="store_true",
                    help="quantiser-only sweep (formats x rounding modes x Hadamard blocks x sizes) "
                         "instead of the layer-set step")
    ap.add_argument("--sweep-log2", default="20,22,24,26,28,30",
                    help="log2 element counts of the sweep tensors (rows of 4096)")
    ap.add_argument("--sweep-cases", default="all",
                    help="comma list of sweep case names (e.g. nvfp4-fos-h0,nvfp4-eden-h128) or 'all'")
    ap.add_argument("--sweep-reps", type=int, default=10)
    ap.add_argument("--diagnostics", action="store_true",
                    help="quantisation MSE (Table 1) and projection magnitude misalignment of every "
                         "mode, computed with the library's kernels; one JSON line per case")
    args = ap.parse_args()
    cfg = dict(CONFIGS[args.config])
    if args.config == 4:
        keep = args.layers.split(",")
        cfg["layers"] = tuple(L for L in LAYERS if L[0] in keep)
    if args.tokens:
        cfg["M"] = args.tokens
    args.cfg = cfg
    return args


# --------------------------------------------------------------- ranks --
def init_dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """Max of a float over all ranks (identity for one rank)."""
    if world <= 1:
        return float(x)
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# -------------------------------------------------------------- clocks --
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            sel = str(self.dev)
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", sel, "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 7:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(r[0]) for r in rows if num(r[0]) is not None]
        pw = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[3 + i].lower().startswith("active")})
        loaded = [s for s, p in zip(sm, pw) if p is not None and p > 300] or sm
        return {"sm_mhz": float(np.median(loaded)) if loaded else None,
                "sm_max_mhz": num(rows[0][1]), "reasons": reasons, "samples": len(rows),
                "power_w_max": max(pw) if pw else None}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def fp4_peak(peaks, src, timed_s):
    """Dense FP4 tensor peak: a measured bf16 GEMM rate times the nominal
    fp4/bf16 ratio; the burst rate for a timed region shorter than
    SUSTAINED_AFTER_S seconds, the power-capped sustained rate otherwise."""
    sustained = timed_s >= SUSTAINED_AFTER_S and "bf16_tflops_sustained" in peaks
    key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    return peaks[key] * FP4_OVER_BF16, "%s cuBLAS bf16 %s %.1f x %.0f (nominal fp4/bf16), timed region %.2f s" % (
        src, "sustained" if sustained else "burst", peaks[key], FP4_OVER_BF16, timed_s)


# ------------------------------------------------------------ workload --
def recipe_preset(api, name):
    return api.recipe({"rtn": api.RECIPE_RTN, "quartet": api.RECIPE_QUARTET,
                       "quartet2": api.RECIPE_QUARTET2}[name])


def layer_data(cfg, li, M, K, N):
    """Seeded bf16 inputs of layer li (uint16 bit patterns): data seed
    cfg["seed"] + li (the layer set's four layers use 3, 4, 5, 6)."""
    r, seed = cfg["recipe"], cfg["seed"] + li
    if r == "rtn":
        d = syn.linear_rtn_small(seed) if (M, K, N) == (256, 512, 512) else {
            "X": syn.gaussian((M, K), 1.0, seed, 0), "W": syn.gaussian((N, K), 0.02, seed, 1)}
        d["dY"] = syn.gaussian((M, N), 1e-3, seed, 2)
        return d
    if r == "quartet":
        return syn.linear_quartet(M, N, K, seed)
    return syn.linear_quartet2(M, N, K, seed)


def make_host_data(cfg):
    """Seeded synthetic bf16 inputs of every layer, in pinned host memory."""
    out = []
    for li, (name, K, N) in enumerate(cfg["layers"]):
        d = layer_data(cfg, li, cfg["M"], K, N)
        out.append({k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).pin_memory()
                    for k, v in d.items()})
    return out


def quant_bytes(api, fmt, rnd, had, src):
    """Algorithmic HBM bytes per quantised element of one quantiser call from
    bf16 (`src` = "bf16": read 2 B) or from a saved FP4 tensor ("fp4": codes
    0.5 + one scale per group): the input read, codes 0.5 and one scale copy
    1/g written; NVFP4 global-amax modes (RTN, 4/6, SR, QuEST) read the input
    a second time (amax pass); QuEST writes a 1-bit mask; MS-EDEN writes and
    re-reads bf16 pseudo-scales (2 x 2/16) and fp32 EDEN factors (2 x 4/had)."""
    g = api.GROUP[fmt]
    rd = 2.0 if src == "bf16" else 0.5 + 1.0 / g
    b = rd + 0.5 + 1.0 / g
    if fmt == api.NVFP4 and rnd != api.MS_EDEN:
        b += rd
    if rnd == api.QUEST:
        b += 1.0 / 8
    if rnd == api.MS_EDEN:
        b += 2 * 2.0 / 16 + 2 * 4.0 / had
    return b


def quant_bytes_per_elem(kind):
    """Per-element bytes of the three quantiser calls of the Quartet II step."""
    from fp4_microscaled_quantized_b200 import api
    if kind == "fos":
        return quant_bytes(api, api.NVFP4, api.FOUR_OVER_SIX, 0, "bf16")
    if kind == "eden":
        return quant_bytes(api, api.NVFP4, api.MS_EDEN, 128, "bf16")
    if kind == "eden_requant":
        return quant_bytes(api, api.NVFP4, api.MS_EDEN, 128, "fp4")
    raise ValueError(kind)


def step_flops(cfg):
    mult = 6.0 if cfg["bwd"] else 2.0
    return sum(mult * cfg["M"] * N * K for _, K, N in cfg["layers"])


class Layers:
    """Device buffers of every layer: inputs, the saved context, outputs,
    the linear entry points' workspaces, and the backward operands the
    instrumented primitive sequence writes."""

    def __init__(self, api, cfg, device, host):
        self.api, self.cfg, self.M = api, cfg, cfg["M"]
        self.r = recipe_preset(api, cfg["recipe"])
        r, M = self.r, self.M
        self.layers = []
        qws = 16
        for li, (name, K, N) in enumerate(cfg["layers"]):
            L = {"name": name, "K": K, "N": N, **{k: v.to(device) for k, v in host[li].items()}}
            L["ctx"] = api.alloc_ctx(r, M, N, K, device)
            L["Y"] = torch.empty((M, N), dtype=torch.float32, device=device)
            if cfg["bwd"]:
                L["dX"] = torch.empty((M, K), dtype=torch.float32, device=device)
                L["dW"] = torch.empty((N, K), dtype=torch.float32, device=device)
                L["wsb"] = api.linear_workspace(r, M, N, K, True, device)
                L["e_row"] = api.alloc_qtensor(M, N, r.fmt, linear=False, device=device)
                L["w_t"] = api.alloc_qtensor(K, N, r.fmt, linear=False, device=device)
                L["e_t"] = api.alloc_qtensor(N, M, r.fmt, linear=False, device=device)
                L["x_t"] = api.alloc_qtensor(K, M, r.fmt, linear=False, device=device)
                for a, b in ((M, N), (K, N), (N, M), (K, M)):
                    qws = max(qws, api.workspace_size(a, b, r.fmt, r.bwd_rounding, r.bwd_had))
            L["wsf"] = api.linear_workspace(r, M, N, K, False, device)
            w_rnd = r.w_rounding if r.w_rounding >= 0 else r.fwd_rounding
            qws = max(qws, api.workspace_size(M, K, r.fmt, r.fwd_rounding, r.fwd_had),
                      api.workspace_size(N, K, r.fmt, w_rnd, r.fwd_had))
            self.layers.append(L)
        self.qws = api.alloc_workspace(qws, device)

    def linear_step(self, step_seed):
        """One step through fp4_linear_fwd / fp4_linear_bwd (the timed `value`)."""
        api, r = self.api, self.r
        for L in self.layers:
            api.linear_fwd(L["X"], L["W"], r, 0, ctx=L["ctx"], Y=L["Y"], ws=L["wsf"])
            if self.cfg["bwd"]:
                api.linear_bwd(L["dY"], L["ctx"], step_seed, dX=L["dX"], dW=L["dW"], ws=L["wsb"])

    def primitive_step(self, step_seed, ev=None):
        """The same kernels through the primitive entry points, in the order
        and with the seeds and tags fp4_linear_fwd / fp4_linear_bwd use, each
        call wrapped by ev(kind, units, fn) (CUDA events) when given."""
        api, r, M, ws = self.api, self.r, self.M, self.qws
        ev = ev or (lambda kind, units, fn: fn())
        fmt = r.fmt
        w_rnd = r.w_rounding if r.w_rounding >= 0 else r.fwd_rounding
        rz = bool(r.bwd_randomized)
        inv_h = r.fwd_had if r.mask_epilogue else 0
        for L in self.layers:
            K, N, ctx = L["K"], L["N"], L["ctx"]
            ev(("q", fmt, r.fwd_rounding, r.fwd_had, "bf16"), M * K,
               lambda: api.quantize(L["X"], fmt, r.fwd_rounding, r.fwd_had, False, 0, 0, TAG_X, out=ctx.xq, ws=ws))
            ev(("q", fmt, w_rnd, r.fwd_had, "bf16"), N * K,
               lambda: api.quantize(L["W"], fmt, w_rnd, r.fwd_had, False, 0, 0, TAG_W, out=ctx.wq, ws=ws))
            ev("gemm", 2.0 * M * N * K, lambda: api.gemm(ctx.xq, ctx.wq, out=L["Y"]))
            if not self.cfg["bwd"]:
                continue
            if r.w_reuse:
                ev(("q", fmt, r.bwd_rounding, 0, "bf16"), M * N,
                   lambda: api.quantize(L["dY"], fmt, r.bwd_rounding, 0, False, step_seed, GEMM_DX, TAG_E_ROW,
                                        out=L["e_row"], ws=ws))
                ev(("t16",), N * K, lambda: api.transpose_square16(ctx.wq, out=L["w_t"]))
            else:
                ev(("q", fmt, r.bwd_rounding, r.bwd_had, "bf16"), M * N,
                   lambda: api.quantize(L["dY"], fmt, r.bwd_rounding, r.bwd_had, rz, step_seed, GEMM_DX,
                                        TAG_E_ROW, out=L["e_row"], ws=ws))
                ev(("q", fmt, r.bwd_rounding, r.bwd_had, "fp4"), N * K,
                   lambda: api.requantize(ctx.wq, r.bwd_rounding, r.bwd_had, rz, step_seed, GEMM_DX, TAG_W_T,
                                          transpose=True, out=L["w_t"], ws=ws))
            ev("gemm", 2.0 * M * N * K,
               lambda: api.gemm(L["e_row"], L["w_t"], out=L["dX"], mask=ctx.xq.mask if inv_h else None,
                                inverse_had=inv_h))
            ev(("q", fmt, r.bwd_rounding, r.bwd_had, "bf16"), M * N,
               lambda: api.quantize(L["dY"], fmt, r.bwd_rounding, r.bwd_had, rz, step_seed, GEMM_DW, TAG_E_T,
                                    transpose=True, out=L["e_t"], ws=ws))
            ev(("q", fmt, r.bwd_rounding, r.bwd_had, "fp4"), M * K,
               lambda: api.requantize(ctx.xq, r.bwd_rounding, r.bwd_had, rz, step_seed, GEMM_DW, TAG_X_T,
                                      transpose=True, out=L["x_t"], ws=ws))
            ev("gemm", 2.0 * M * N * K,
               lambda: api.gemm(L["e_t"], L["x_t"], out=L["dW"], mask=ctx.wq.mask if inv_h else None,
                                inverse_had=inv_h))


class Recorder:
    """CUDA events around every primitive call (on the current stream, the
    one the library launches on)."""

    def __init__(self):
        self.records = []

    def __call__(self, kind, units, fn):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        self.records.append((kind, units, a, b))

    def summary(self, api):
        g_t = g_f = q_t = q_b = 0.0
        n_gemm = 0
        for kind, units, a, b in self.records:
            ms = a.elapsed_time(b)
            if kind == "gemm":
                g_t += ms
                g_f += units
                n_gemm += 1
            elif kind[0] == "t16":                   # square-block transpose: FP4 in and out
                q_t += ms
                q_b += units * 2 * (0.5 + 1 / 16)
            else:
                q_t += ms
                q_b += units * quant_bytes(api, *kind[1:])
        return {"gemm_ms": g_t, "gemm_flops": g_f, "n_gemm": n_gemm, "quant_ms": q_t, "quant_bytes": q_b}


def timed(run, steps, flush):
    """Device time (ms) of `steps` calls of run(k): one event pair around all
    of them, or, with an L2 flush between steps (inputs smaller than L2), the
    sum of per-step event pairs with the flush outside them."""
    if flush is None:
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for k in range(steps):
            run(k)
        e.record()
        torch.cuda.synchronize()
        return s.elapsed_time(e)
    pairs = []
    for k in range(steps):
        flush.zero_()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        run(k)
        e.record()
        pairs.append((s, e))
    torch.cuda.synchronize()
    return sum(s.elapsed_time(e) for s, e in pairs)


def run_e2e(api, cfg, steps, device, host):
    """The same metric through the public linear-layer API with host buffers:
    every step copies X, W, dY of every layer host->device (pinned), runs
    fp4_linear_fwd (+ fp4_linear_bwd) and reads the parameter gradient dW
    (Y for the forward-only config) back device->host; Y and dX stay on the
    device, where the next layer of a network consumes them.  The copies run
    on their own streams, overlapped with the other layers' compute."""
    r = recipe_preset(api, cfg["recipe"])
    M = cfg["M"]
    out_key = "dW" if cfg["bwd"] else "Y"
    devbuf = []
    for li, (name, K, N) in enumerate(cfg["layers"]):
        d = host[li]
        b = {"X": torch.empty_like(d["X"], device=device), "W": torch.empty_like(d["W"], device=device),
             "dY": torch.empty_like(d["dY"], device=device), "ctx": api.alloc_ctx(r, M, N, K, device),
             "Y": torch.empty((M, N), dtype=torch.float32, device=device),
             "wsf": api.linear_workspace(r, M, N, K, False, device)}
        if cfg["bwd"]:
            b.update({"dX": torch.empty((M, K), dtype=torch.float32, device=device),
                      "dW": torch.empty((N, K), dtype=torch.float32, device=device),
                      "wsb": api.linear_workspace(r, M, N, K, True, device)})
        b["host_out"] = torch.empty(b[out_key].shape, dtype=torch.float32).pin_memory()
        devbuf.append(b)
    in_keys = ("X", "W", "dY") if cfg["bwd"] else ("X", "W")
    h2d = sum(h[k].numel() * h[k].element_size() for h in host for k in in_keys)
    d2h = sum(b[out_key].numel() * 4 for b in devbuf)

    comp = torch.cuda.current_stream()
    cin, cout = torch.cuda.Stream(), torch.cuda.Stream()
    n = len(devbuf)
    ev_in = [torch.cuda.Event() for _ in range(n)]
    ev_done = [torch.cuda.Event() for _ in range(n)]
    ev_d2h = [torch.cuda.Event() for _ in range(n)]
    ev_out = torch.cuda.Event()

    def step(seed, first):
        for i, (h, b) in enumerate(zip(host, devbuf)):
            with torch.cuda.stream(cin):
                if not first:
                    cin.wait_event(ev_done[i])
                for k in in_keys:
                    b[k].copy_(h[k], non_blocking=True)
                ev_in[i].record(cin)
        for i, b in enumerate(devbuf):
            comp.wait_event(ev_in[i])
            if not first:
                comp.wait_event(ev_d2h[i])         # last step's output has left this buffer
            api.linear_fwd(b["X"], b["W"], r, 0, ctx=b["ctx"], Y=b["Y"], ws=b["wsf"])
            if cfg["bwd"]:
                api.linear_bwd(b["dY"], b["ctx"], seed, dX=b["dX"], dW=b["dW"], ws=b["wsb"])
            ev_done[i].record(comp)
            with torch.cuda.stream(cout):
                cout.wait_event(ev_done[i])
                b["host_out"].copy_(b[out_key], non_blocking=True)
                ev_d2h[i].record(cout)
        ev_out.record(cout)

    step(0, True)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(comp)
    for k in range(steps):
        step(100 + k, k == 0)
    comp.wait_event(ev_out)                      # the last output is on the host
    e.record(comp)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    del devbuf
    torch.cuda.empty_cache()
    return {"value": step_flops(cfg) / (ms * 1e-3) / 1e12, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": ms, "steps": steps,
            "to_host": out_key + " of every layer", "stays_on_device": "Y, dX" if cfg["bwd"] else ""}


# ------------------------------------------------------ quantiser sweep --
SWEEP_COLS = 4096
RND_NAMES = {0: "rtn", 1: "quest", 2: "fos", 3: "sr", 4: "eden", 5: "rtn16x16"}


def sweep_cases(api):
    """(name, fmt, rounding, had_block, randomized) of every combination the C ABI
    accepts: MXFP4 (RTN, QuEST, SR) and NVFP4 (RTN, QuEST, 4/6, SR) with Hadamard
    none/16/32/64/128/256, NVFP4 MS-EDEN with 16/32/64/128/256, NVFP4 RTN with
    16 x 16 block scales.  The stochastic modes use the
    randomized transform (backward pass), the others the deterministic one."""
    out = []
    for fmt, fname, rnds in ((api.MXFP4, "mxfp4", (api.RTN, api.QUEST, api.SR)),
                             (api.NVFP4, "nvfp4", (api.RTN, api.QUEST, api.FOUR_OVER_SIX, api.SR,
                                                   api.MS_EDEN))):
        for rnd in rnds:
            for had in (0, 16, 32, 64, 128, 256):
                if rnd == api.MS_EDEN and had == 0:
                    continue
                rand = rnd in (api.SR, api.MS_EDEN) and had > 0
                out.append(("%s-%s-h%d" % (fname, RND_NAMES[rnd], had), fmt, rnd, had, rand))
    out.append(("nvfp4-rtn16x16-h0", api.NVFP4, api.RTN_SQUARE16, 0, False))
    # the MSE-optimal scale search (fp4_quantize_mse) with 0 and 2 alternations
    out.append(("nvfp4-mse-i0-h0", api.NVFP4, "mse0", 0, False))
    out.append(("nvfp4-mse-i2-h0", api.NVFP4, "mse2", 0, False))
    # forward-only transforms: a DCT-II / DST-II block transform (fp32 out)
    # quantised by fp4_quantize_f32, and MXFP4 with fitted scales
    for kind, k, fmt, fname in (("dct2", 32, api.NVFP4, "nvfp4"), ("dct2", 128, api.NVFP4, "nvfp4"),
                                ("dst2", 256, api.MXFP4, "mxfp4")):
        out.append(("%s-rtn-%s-k%d" % (fname, kind, k), fmt, ("xform", kind, k), k, False))
    for had in (0, 32):
        out.append(("mxfp4-fit-h%d" % had, api.MXFP4, ("fit",), had, False))
    return out


def sweep_bytes_per_elem(api, fmt, rnd, had):
    """Algorithmic HBM bytes per element of one quantise call from bf16 (see
    quant_bytes); the 16 x 16 square-block mode reads the input twice (block
    maxima); the MSE search ("mseI", I alternations) reads the input once for
    the amax and once per group step, writing codes and scales each time."""
    if isinstance(rnd, str):
        return 2.0 + (int(rnd[3:]) + 1) * (2.0 + 0.5 + 1.0 / 16)
    if isinstance(rnd, tuple) and rnd[0] == "xform":
        # bf16 read + fp32 write, then the fp32 quantiser: (amax read 4 for NVFP4) + read 4 + codes + scales
        return 2.0 + 4.0 + (4.0 if fmt == api.NVFP4 else 0.0) + 4.0 + 0.5 + (1.0 / 16 if fmt == api.NVFP4 else 1.0 / 32)
    if isinstance(rnd, tuple) and rnd[0] == "fit":
        # range pass read 2, quantise pass read 2 + codes 0.5 + one level byte per 32
        return 2.0 + 2.0 + 0.5 + 1.0 / 32
    return quant_bytes(api, fmt, rnd, had, "bf16")


def quant_sweep(args):
    """Config-5 sweep: every quantiser combination on N(0,1) + 0.1% x50
    outlier tensors of 2^n bf16 elements (rows of 4096), row-wise.  Each call
    is timed alone with CUDA events on the launching stream, the L2 flushed
    (a 256 MiB write) before every repetition; one JSON line per case."""
    from fp4_microscaled_quantized_b200 import api
    api.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, src = load_peaks()
    logs = [int(s) for s in args.sweep_log2.split(",")]
    cases = sweep_cases(api)
    if args.sweep_cases != "all":
        keep = set(args.sweep_cases.split(","))
        cases = [c for c in cases if c[0] in keep]
    rows_max = (1 << max(logs)) // SWEEP_COLS
    # One seeded tensor of up to 2^28 elements; smaller sizes are its leading
    # rows, larger ones repeat it (host generation of 2^30 draws takes minutes).
    rows_gen = min(rows_max, (1 << 28) // SWEEP_COLS)
    bits = syn.outlier_elements((rows_gen, SWEEP_COLS), seed=7)
    x_gen = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)
    del bits
    x_all = x_gen.repeat((rows_max + rows_gen - 1) // rows_gen, 1)[:rows_max] if rows_max > rows_gen else x_gen
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    for lg in logs:
        rows = (1 << lg) // SWEEP_COLS
        x = x_all[:rows]
        for name, fmt, rnd, had, rand in cases:
            out = api.alloc_qtensor(rows, SWEEP_COLS, fmt, linear=False, mask=(rnd == api.QUEST),
                                    device=dev)
            if isinstance(rnd, str):
                ws = api.alloc_workspace(api.quantize_mse_workspace_size(rows, SWEEP_COLS), dev)
                call = lambda s, it=int(rnd[3:]): api.quantize_mse(x, it, out=out, ws=ws)  # noqa: E731
            elif isinstance(rnd, tuple) and rnd[0] == "xform":
                y = torch.empty((rows, SWEEP_COLS), dtype=torch.float32, device=dev)
                ws = api.alloc_workspace(max(api.workspace_size(rows, SWEEP_COLS, fmt, api.RTN, 0), 4 * had * had), dev)
                kind = api.XFORM_DCT2 if rnd[1] == "dct2" else api.XFORM_DST2

                def call(s, kind=kind, y=y, ws=ws, out=out):
                    api.block_transform(x, kind, had, out=y, ws=ws)
                    api.quantize_f32(y, fmt, api.RTN, s, 1, linear=False, out=out, ws=ws)
            elif isinstance(rnd, tuple) and rnd[0] == "fit":
                ws = api.alloc_workspace(api.quantize_mx_fit_workspace_size(), dev)
                fit = api.FitTensor(torch.empty((rows, SWEEP_COLS // 2), dtype=torch.uint8, device=dev),
                                    torch.empty((rows, SWEEP_COLS // 32), dtype=torch.uint8, device=dev),
                                    torch.empty((256,), dtype=torch.float32, device=dev))
                call = lambda s, h=had, ws=ws, fit=fit: api.quantize_mx_fit(x, h, ws=ws, out=fit)  # noqa: E731
            else:
                ws = api.alloc_workspace(api.workspace_size(rows, SWEEP_COLS, fmt, rnd, had), dev)
                call = lambda s: api.quantize(x, fmt, rnd, had, rand, s, 0, 1, out=out, ws=ws)  # noqa: E731
            lc0 = api.launch_count()
            for w in range(3):
                call(w)
            launches = (api.launch_count() - lc0) // 3
            ts = []
            for k in range(args.sweep_reps):
                flush.zero_()
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                call(100 + k)
                b.record(stream)
                b.synchronize()
                ts.append(a.elapsed_time(b))
            ms = float(np.median(ts))
            n = rows * SWEEP_COLS
            gbs = n * sweep_bytes_per_elem(api, fmt, rnd, had) / (ms * 1e-3) / 1e9
            print(json.dumps({"case": name, "log2_elems": lg, "elems": n, "us": round(ms * 1e3, 2),
                              "gb_s": round(gbs, 1), "hbm_frac": round(gbs / peaks["hbm_gbs"], 3),
                              "bytes_per_elem": sweep_bytes_per_elem(api, fmt, rnd, had),
                              "launches": int(launches), "peak": "%s copy %.0f GB/s" % (src, peaks["hbm_gbs"])}),
                  flush=True)
            del out, ws
    if api.get_last_error() != 0:
        raise SystemExit("device status %d after the sweep" % api.get_last_error())


# --------------------------------------------------------- CPU oracle --
def oracle_recipe(cfg):
    from oracle import linear as ln
    return {"rtn": ln.RTN, "quartet": ln.QUARTET, "quartet2": ln.QUARTET2}[cfg["recipe"]]


def oracle_sample(cfg, n_rows, n_out, seed=0):
    """The oracle's step on a bounded sample of the workload: the first
    n_rows tokens and n_out output features of the config's first layer (its
    full K), forward + backward (forward only for config 1).  Single-threaded
    numpy (BLAS limited to one thread).  Returns (flops, seconds)."""
    from threadpoolctl import threadpool_limits
    from oracle import linear as ln
    K = cfg["layers"][0][1]
    d = layer_data(dict(cfg, M=n_rows), seed, n_rows, K, n_out)
    f = syn.bf16_bits_to_f32
    rec = oracle_recipe(cfg)
    with threadpool_limits(1):
        t0 = time.perf_counter()
        _, _, ctx = ln.linear_fwd(f(d["X"]), f(d["W"]), rec)
        if cfg["bwd"]:
            ln.linear_bwd(f(d["dY"]), ctx, rec, 7)
        dt = time.perf_counter() - t0
    flops = (6.0 if cfg["bwd"] else 2.0) * n_rows * n_out * K
    return flops, dt


def _oracle_worker(job):
    """One all-core worker: the oracle sample, timed by the host's wall clock
    so the workers' intervals can be combined."""
    cfg, n_rows, n_out, seed = job
    t0 = time.time()
    f, dt = oracle_sample(cfg, n_rows, n_out, seed)
    return f, dt, t0, time.time()


def host_cpu():
    """The host's CPU model and logical core count, recorded beside the oracle's timing."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return "%s, %d logical cores" % (model, os.cpu_count() or 0)


def sample_shape(cfg, target_s):
    """(rows, output features) of an oracle sample that takes about
    target_s seconds on one core (calibrated on a small sample)."""
    n_rows = min(128, cfg["M"])
    N = cfg["layers"][0][2]
    f0, t0 = oracle_sample(cfg, n_rows, min(128, N))
    n_out = int(min(N, max(128, 128 * target_s / max(t0, 1e-3))) // 128 * 128)
    return n_rows, max(n_out, min(128, N))


def cpu_baseline(cfg, target_s=12.0):
    """The oracle on the host's cores: one sample single-threaded, then the
    same sample in one spawned process per logical core at once (each
    single-threaded numpy, different seeds); the all-core value is the total
    flops over the wall time from the first start to the last end."""
    import concurrent.futures as cf
    import multiprocessing as mp
    n_rows, n_out = sample_shape(cfg, target_s)
    f1, t1 = oracle_sample(cfg, n_rows, n_out)
    cores = os.cpu_count() or 1
    ctx = mp.get_context("spawn")
    small = (cfg, n_rows, min(128, cfg["layers"][0][2]), 0)
    with cf.ProcessPoolExecutor(max_workers=cores, mp_context=ctx) as ex:
        list(ex.map(_oracle_worker, [small] * cores))        # every worker imports numpy and the oracle first
        res = list(ex.map(_oracle_worker, [(cfg, n_rows, n_out, k) for k in range(cores)]))
    tot_f = sum(r[0] for r in res)
    wall = max(r[3] for r in res) - min(r[2] for r in res)
    sample = "%s: first layer, %d tokens x %d output features x K=%d, %s (quantisers + fp64 GEMMs)" % (
        cfg["recipe"], n_rows, n_out, cfg["layers"][0][1], "fwd+bwd" if cfg["bwd"] else "fwd")
    return {"value": tot_f / wall / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": sample + "; one sample per core in %d spawned processes, %.1f s wall" % (cores, wall),
            "single_thread": {"value": f1 / t1 / 1e12, "unit": UNIT, "cores": 1, "seconds": round(t1, 2)},
            "host": host_cpu()}


def reference_arm(args, world, rank):
    """The oracle timed on the host cores on this config's workload, a
    bounded sample per step (the pages hold no code to run)."""
    if rank != 0:
        return
    cfg = args.cfg
    per_step = max(3.0, 150.0 / max(1, args.steps + args.warmup))
    n_rows, n_out = sample_shape(cfg, per_step)
    for _ in range(args.warmup):
        oracle_sample(cfg, n_rows, n_out)
    tot_f = tot_t = 0.0
    for k in range(args.steps):
        f, t = oracle_sample(cfg, n_rows, n_out, seed=k)
        tot_f += f
        tot_t += t
    v = tot_f / tot_t / 1e12
    sample = "%s: first layer, %d tokens x %d output features x K=%d per step, %s" % (
        cfg["recipe"], n_rows, n_out, cfg["layers"][0][1], "fwd+bwd" if cfg["bwd"] else "fwd")
    print(json.dumps({
        "metric": METRIC, "value": v, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32 quantisers, f64 GEMM",
        "data": "synthetic", "config": config_dict(cfg),
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample,
                         "host": host_cpu()},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))


def config_dict(cfg):
    rec = {"rtn": "NVFP4 RTN fwd", "quartet": "quartet: MXFP4 QuEST+H32 fwd, SR(3/4 RHT32) bwd, mask/H32^-1",
           "quartet2": "quartet2: NVFP4 RTN+4/6 fwd, RHT128 + MS-EDEN bwd"}[cfg["recipe"]]
    l2 = ("L2 flushed (256 MiB write) between timed steps" if cfg["flush"] else
          "inputs larger than L2 (about 9 GB touched per step)")
    return {"workload": cfg["workload"], "tokens": cfg["M"], "recipe": rec,
            "outputs": "fp32 Y" + (", dX, dW" if cfg["bwd"] else ""), "global_batch": cfg["M"], "l2": l2,
            "parallelism": "replicas"}


# ------------------------------------------------------------------ main --
def main():
    args = parse()
    world, rank, local = init_dist()
    if args.impl == "reference":
        reference_arm(args, world, rank)
        return
    if args.quant_sweep:
        if rank == 0:
            quant_sweep(args)
        return
    if args.diagnostics:
        if rank == 0:
            from fp4_microscaled_quantized_b200 import api, diagnostics
            api.load()
            for row in diagnostics.table(torch.device("cuda", local)):
                print(json.dumps(row), flush=True)
        return
    from fp4_microscaled_quantized_b200 import api
    api.load()
    cfg = args.cfg
    dev = torch.device("cuda", local)
    t_gen = time.perf_counter()
    host = make_host_data(cfg)
    t_gen = time.perf_counter() - t_gen
    L = Layers(api, cfg, dev, host)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev) if cfg["flush"] else None
    warm = max(args.warmup, 3)
    for w in range(warm):
        L.linear_step(1000 + w)
        L.primitive_step(1000 + w)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()

    # timed region 1: `value`, through fp4_linear_fwd / fp4_linear_bwd alone
    clocks = ClockSampler(local)
    clocks.start()
    lc0 = api.launch_count()
    total_ms = timed(L.linear_step, args.steps, flush)
    lc1 = api.launch_count()
    barrier(world)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = total_ms / args.steps
    ms_max = max_over_ranks(ms, world)
    value = world * step_flops(cfg) / (ms_max * 1e-3) / 1e12

    # timed region 2: the same kernels through the primitive entry points,
    # CUDA events around every call (per-kernel split and roofline)
    rec = Recorder()
    inst_ms = timed(lambda k: L.primitive_step(k, rec), args.steps, flush) / args.steps
    st = rec.summary(api)
    err = api.get_last_error()

    peaks, src = load_peaks()
    peak, peak_src = fp4_peak(peaks, src, total_ms * 1e-3)
    g_ach = st["gemm_flops"] / (st["gemm_ms"] * 1e-3) / 1e12
    q_ach = st["quant_bytes"] / (st["quant_ms"] * 1e-3) / 1e9
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "gemm_traffic.json")
    if args.config == 4 and os.path.exists(tpath):
        trec = json.load(open(tpath))
        gemm_src = os.path.join(ROOT, "fp4_microscaled_quantized_b200", "csrc", "gemm_sm100.cu")
        # counters taken on another version of the kernel do not describe this one
        if trec.get("kernel_source_sha256") == hashlib.sha256(open(gemm_src, "rb").read()).hexdigest():
            traffic = trec.get("bytes_per_launch")
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": warm, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("mxfp4 (e2m1 x e2m1, e8m0 scales, fp32 accumulate)" if cfg["recipe"] == "quartet" else
                  "nvfp4 (e2m1 x e2m1, e4m3 scales, fp32 accumulate)"),
        "data": "synthetic (seeded; Gaussian / Student-t / outlier distributions of the pages' workloads)",
        "config": config_dict(cfg),
        "roofline": {"bound": "tensor", "achieved": g_ach, "peak": peak, "unit": "TFLOP/s",
                     "frac": g_ach / peak, "traffic": traffic,
                     "kernel": "k_gemm_pair (tcgen05 cta_group::2 %s)" % (
                         "mxf4nvf4" if cfg["recipe"] != "quartet" else "mxf4") if cfg["M"] > 128 else
                     "k_gemm (tcgen05 cta_group::1)",
                     "peak_source": peak_src},
        "quantizers": {"achieved": q_ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                       "frac": q_ach / peaks["hbm_gbs"], "share_of_step": st["quant_ms"] / (inst_ms * args.steps),
                       "peak_source": src + " copy bandwidth"},
        "gemm_share_of_step": st["gemm_ms"] / (inst_ms * args.steps),
        "instrumented_ms_per_step": inst_ms,
        "end_to_end_frac_of_fp4_peak": value / world / peak,
        "clocks": clk, "gpu_launches": int(lc1 - lc0), "device_status": err,
        "input_generation_s": round(t_gen, 1),
    }
    if args.config == 1:
        out["latency_us"] = ms_max * 1e3
    del L
    torch.cuda.empty_cache()
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        out["cpu_baseline"] = cpu_baseline(cfg)
    if args.e2e_steps > 0:
        e2e = run_e2e(api, cfg, args.e2e_steps, dev, host)
        e2e["value"] = world * e2e["value"] * (e2e["ms_per_step"] / max_over_ranks(e2e["ms_per_step"], world))
        out["e2e"] = e2e
    if rank == 0:
        print(json.dumps(out))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
