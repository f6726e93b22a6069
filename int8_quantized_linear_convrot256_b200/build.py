"""Builds libck.so in-tree with nvcc for sm_100a (B200) only.

    python int8_quantized_linear_convrot256_b200/build.py [--force] [--verbose] [--checked]

(run as a script: importing the package itself needs a built libck.so)

Each .cu under csrc/ is compiled to an object under _build/, then linked into
int8_quantized_linear_convrot256_b200/libck.so with the CUDA runtime linked
statically, so the library needs nothing from the CUDA toolkit at run time
except the driver. The quantiser is compiled with -fmad=false (no contraction
of a multiply and an add into an FMA) and none of the units uses fast math or
flush-to-zero, so every fp32 operation rounds as IEEE round-to-nearest-even.
--checked builds libck_checked.so instead (objects under _build/checked/):
the same sources with CK_CHECKED defined, which compiles in the kernels'
device-side index checks (see ck_checked_violations in include/ck.h).
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libck.so")
LIB_CHECKED = os.path.join(PKG, "libck_checked.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
          "--expt-relaxed-constexpr", f"-I{INCLUDE}", f"-I{CSRC}",
          "-ftz=false", "-prec-div=true", "-prec-sqrt=true"]
PER_FILE = {
    "quant_rotate.cu": ["-fmad=false"],
    "dequant.cu": ["-fmad=false"],
}
SOURCES = ["api.cu", "quant_rotate.cu", "gemm_i8_tcgen05.cu", "gemm_nvfp4_tcgen05.cu", "noalloc.cu",
           "dequant.cu", "rmsnorm.cu"]
HEADERS = ["ck_device.cuh", "internal.h", "libck.map"]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libck.so")
    return cand


def _newest_dep_mtime() -> float:
    paths = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "ck.h"), __file__]
    return max(os.path.getmtime(p) for p in paths)


def _compile(src: str, verbose: bool, force: bool, ptxas_v: bool, checked: bool = False) -> str:
    build_dir = os.path.join(BUILD, "checked") if checked else BUILD
    obj = os.path.join(build_dir, src.replace(".cu", ".o"))
    srcp = os.path.join(CSRC, src)
    if (not force and os.path.exists(obj)
            and os.path.getmtime(obj) >= max(os.path.getmtime(srcp), _newest_dep_mtime())):
        return obj
    cmd = [nvcc(), *ARCH, *COMMON, *PER_FILE.get(src, []), *(["-DCK_CHECKED"] if checked else []),
           "-c", srcp, "-o", obj]
    if ptxas_v:
        cmd += ["-Xptxas", "-v"]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    if (verbose or ptxas_v) and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, flush=True)
    return obj


def build(force: bool = False, verbose: bool = False, ptxas_v: bool = False,
          checked: bool = False) -> str:
    """Builds libck.so, or with checked=True libck_checked.so (the kernels'
    index checks compiled in: CK_CHECKED)."""
    lib = LIB_CHECKED if checked else LIB
    os.makedirs(os.path.join(BUILD, "checked") if checked else BUILD, exist_ok=True)
    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, force, ptxas_v, checked), SOURCES))
    if (force or not os.path.exists(lib)
            or os.path.getmtime(lib) < max(os.path.getmtime(o) for o in objs)):
        tmp = lib + f".tmp{os.getpid()}"
        cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", *objs, "-o", tmp,
               "-Xlinker", "--no-undefined", "-Xlinker", f"--version-script={os.path.join(CSRC, 'libck.map')}",
               "-ldl", "-lrt", "-lpthread"]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib)
    return lib


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true", help="print registers/spills per kernel")
    ap.add_argument("--checked", action="store_true",
                    help="build libck_checked.so (device-side index checks, CK_CHECKED)")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=a.verbose, ptxas_v=a.ptxas_v, checked=a.checked))
    return 0


if __name__ == "__main__":
    sys.exit(main())
