"""Build libfusednorm.so in-tree with nvcc for sm_100a.

The library is the product: the binding loads it from this directory and
refuses to run without it.  IEEE division and square root, no flush-to-zero
and no fast-math, because the quantized codes are specified bit-exactly.
The twelve (mode, partial-bound) kernel units compile in parallel.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libfusednorm.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + [
    "-lineinfo", "-O3", "-std=c++17",
    "-ftz=false", "-prec-div=true", "-prec-sqrt=true", "-fmad=true",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
]

# one unit per (quantization mode, partial-count bound, row format: 0 bf16, 1 binary16)
UNITS = [("fusednorm", "fusednorm.cu", [])] + [
    (f"rq_{mode}_{maxp}_{io}", "rq_inst.cu",
     [f"-DFN_INST_MODE={mode}", f"-DFN_INST_MAXP={maxp}", f"-DFN_INST_IO={io}"])
    for mode in (0, 1, 2) for maxp in (1, 2, 4, 8) for io in (0, 1)
] + [(f"ar_{mode}", "ar_inst.cu", [f"-DFN_INST_MODE={mode}"]) for mode in (0, 1, 2)] + [
    ("hc", "hc_inst.cu", [])]


def deps():
    return [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh", ".h"))] + \
        [os.path.join(INCLUDE, "fusednorm.h"), os.path.abspath(__file__)]


def nvcc() -> str:
    cand = os.environ.get("NVCC") or "/usr/local/cuda/bin/nvcc"
    return cand if os.path.exists(cand) else "nvcc"


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in deps())


def _compile(unit, extra, verbose):
    name, src, defs = unit
    obj = os.path.join(BUILD, name + ".o")
    cmd = [nvcc(), *NVCC_FLAGS, *extra, *defs, "-I", INCLUDE, "-I", CSRC, "-c", "-o", obj,
           os.path.join(CSRC, src)]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    r = subprocess.run(cmd, capture_output=True, text=True)
    return obj, r


def build_library(force: bool = False, verbose: bool = False, extra=()) -> str:
    if not force and up_to_date() and not extra:
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    jobs = max(1, min(len(UNITS), os.cpu_count() or 1))
    with ThreadPoolExecutor(jobs) as ex:
        results = list(ex.map(lambda u: _compile(u, extra, verbose), UNITS))
    for obj, r in results:
        if r.returncode != 0 or (verbose and r.stderr):
            sys.stderr.write(r.stdout + r.stderr)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {obj}")
    tmp = LIB + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "--cudart", "static", "-o", tmp, *[o for o, _ in results]]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build_library(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                  extra=("-Xptxas", "-v") if "--ptxas-v" in sys.argv else ())
    print(LIB)
