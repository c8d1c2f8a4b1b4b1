"""Build the in-tree C-ABI library ``libfp4_b200.so`` for sm_100a with nvcc.

Each ``csrc/*.cu`` compiles to an object in ``_build/`` (in parallel, rebuilt
when a source or header is newer), then all link into one shared library next
to this file.  The quantiser, C-ABI and block-transform sources build with
``-fmad=false`` so no fp32 multiply-add is ever contracted (the arithmetic
contract with the oracle).
"""
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build", "fp4_b200")
LIB = os.path.join(HERE, "libfp4_b200.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O3",
                 "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def _flags(src):
    extra = []
    name = os.path.basename(src)
    if name.startswith("quant") or name in ("capi.cu", "transform.cu"):
        extra += ["-fmad=false"]
    return COMMON + extra


def _needs(obj, deps):
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose=False, jobs=None):
    os.makedirs(BUILD, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))
    todo = []
    objs = []
    for s in srcs:
        o = os.path.join(BUILD, os.path.basename(s)[:-3] + ".o")
        objs.append(o)
        if _needs(o, [s] + headers):
            todo.append((s, o))

    def one(so):
        s, o = so
        cmd = [NVCC] + _flags(s) + ["-c", s, "-o", o]
        r = subprocess.run(cmd, capture_output=True, text=True)
        return s, r, cmd

    if todo:
        with cf.ThreadPoolExecutor(max_workers=jobs or os.cpu_count()) as ex:
            for s, r, cmd in ex.map(one, todo):
                if verbose or r.returncode:
                    sys.stderr.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
                if r.returncode:
                    raise RuntimeError("nvcc failed on %s" % s)
    if todo or not os.path.exists(LIB) or any(os.path.getmtime(o) > os.path.getmtime(LIB) for o in objs):
        cmd = [NVCC] + ARCH + ["-shared", "-o", LIB] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode:
            sys.stderr.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
            raise RuntimeError("link failed")
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
