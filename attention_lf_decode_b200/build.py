"""Build the sm_100a shared library ``liblf_decode.so`` in-tree with nvcc.

    python -m attention_lf_decode_b200.build [--force] [--verbose] [--ptxas]

The library exports the C ABI of ``include/lf_decode.h``.  The fused kernel's
variants (KV storage x kernel mode) are separate translation units, one
object each from ``csrc/lf_inst.cu``, compiled in parallel and linked with
``csrc/lf_decode.cu``.  The CUDA runtime is linked statically, so the library
does not depend on the runtime version torch ships.  nvcc cross-compiles
without a GPU.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "liblf_decode.so")
OBJDIR = os.path.join(PKG, "_build")
SOURCES = ["lf_decode.cu", "lf_inst.cu"]
HEADERS = ["lf_kernel.cuh", "lf_internal.h", "lf_ptx.cuh"]
# (bytes per cached element, kernel mode) of every compiled variant
VARIANTS = [(2, 0), (2, 1), (2, 2), (1, 0), (1, 1), (1, 2)]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
          "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _newest_input() -> float:
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "lf_decode.h"))
    files.append(os.path.abspath(__file__))
    return max(os.path.getmtime(f) for f in files)


def _units():
    """(source, object, extra flags) of every translation unit."""
    units = [("lf_decode.cu", "lf_decode.o", [])]
    for kvb, mode in VARIANTS:
        units.append(("lf_inst.cu", f"lf_inst_kv{kvb}_m{mode}.o",
                      [f"-DLF_KVB={kvb}", f"-DLF_MODE={mode}"]))
    return units


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    """Compile the library if it is missing or older than its sources."""
    if not force and not ptxas_info and os.path.exists(LIB) and \
            os.path.getmtime(LIB) >= _newest_input():
        return LIB
    os.makedirs(OBJDIR, exist_ok=True)
    base = [nvcc(), *ARCH, *CFLAGS, "-I", INCLUDE, "-I", CSRC]
    if ptxas_info:
        base += ["-Xptxas", "-v"]

    def compile_one(unit):
        src, obj, extra = unit
        cmd = base + extra + ["-c", os.path.join(CSRC, src), "-o", os.path.join(OBJDIR, obj)]
        if verbose:
            print(" ".join(cmd), flush=True)
        return subprocess.run(cmd, capture_output=True, text=True)

    units = _units()
    with ThreadPoolExecutor(max_workers=min(len(units), os.cpu_count() or 1)) as ex:
        results = list(ex.map(compile_one, units))
    for (src, obj, extra), res in zip(units, results):
        if res.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src} {' '.join(extra)}:\n" + res.stdout + res.stderr)
        if verbose or ptxas_info:
            sys.stdout.write(res.stdout + res.stderr)
    tmp = LIB + ".tmp"
    link = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-Xcompiler", "-fPIC",
            *[os.path.join(OBJDIR, obj) for _, obj, _ in units], "-o", tmp]
    res = subprocess.run(link, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc link failed:\n" + res.stdout + res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv or "--ptxas" in sys.argv,
          verbose="--verbose" in sys.argv, ptxas_info="--ptxas" in sys.argv)
    print(LIB)
