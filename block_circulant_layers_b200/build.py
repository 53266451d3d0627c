"""Build the in-tree native libraries of the package.

    python -m block_circulant_layers_b200.build [--force] [--no-emulator]

* librdfft.so         -- the C ABI of include/rdfft.h with the sm_100a kernels
                         (nvcc -gencode arch=compute_100a,code=sm_100a; cross-compiles
                         on a machine without a GPU).
* librdfft_hostemu.so -- the same per-thread rdFFT pass code compiled for the host
                         (g++), used by the CPU tests to check the kernels' index
                         logic and arithmetic without a GPU.

Both land next to this file so that they travel with the source tree.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
GEN = os.path.join(CSRC, "_gen")
BUILD = os.path.join(PKG, "_build")
INCLUDE = os.path.join(ROOT, "include")

LIB = os.path.join(PKG, "librdfft.so")
EMU = os.path.join(PKG, "librdfft_hostemu.so")

CU_SOURCES = ["rdfft_api.cu", "rdfft_kernels.cu", "rdfft2d_kernels.cu", "convert_kernels.cu", "circ_launch.cu",
              "circ_tc.cu", "circ_bwd_fused.cu"] + [
    f"circ_p{p}.cu" for p in (64, 128, 256, 512, 1024, 2048, 4096)]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build librdfft.so")


def _newest_input_mtime() -> float:
    paths = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    paths += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    paths.append(os.path.abspath(__file__))
    return max(os.path.getmtime(p) for p in paths if os.path.isfile(p))


def _up_to_date(target: str) -> bool:
    return os.path.exists(target) and os.path.getmtime(target) >= _newest_input_mtime()


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"command failed ({r.returncode}): {' '.join(cmd)}\n{r.stdout}")
    return r.stdout


def generate() -> None:
    os.makedirs(GEN, exist_ok=True)
    out = os.path.join(GEN, "twiddles.inc")
    gen = os.path.join(CSRC, "gen_twiddles.py")
    if not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(gen):
        _run([sys.executable, gen, out], False)


def build_lib(force=False, verbose=False, ptxas_info=False) -> str:
    if not force and _up_to_date(LIB):
        return LIB
    generate()
    os.makedirs(BUILD, exist_ok=True)
    nvcc = _nvcc()
    flags = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
             "-I", INCLUDE, "-I", CSRC, "-I", GEN] + ARCH
    if ptxas_info:
        flags += ["-Xptxas", "-v"]
    objs = []
    cmds = []
    for src in CU_SOURCES:
        obj = os.path.join(BUILD, src.replace(".cu", ".o"))
        objs.append(obj)
        cmds.append([nvcc, "-c", os.path.join(CSRC, src), "-o", obj] + flags)
    with cf.ThreadPoolExecutor(max_workers=min(len(cmds), os.cpu_count() or 4)) as ex:
        outs = list(ex.map(lambda c: _run(c, verbose), cmds))
    if ptxas_info:
        for o in outs:
            print(o)
    tmp = LIB + ".tmp"
    _run([nvcc, "-shared", "-o", tmp] + objs + ARCH + ["-Xcompiler", "-fPIC"], verbose)
    os.replace(tmp, LIB)
    return LIB


def build_emulator(force=False, verbose=False) -> str:
    if not force and _up_to_date(EMU):
        return EMU
    generate()
    cxx = shutil.which("g++") or "g++"
    tmp = EMU + ".tmp"
    _run([cxx, "-O2", "-std=c++17", "-shared", "-fPIC", "-ffp-contract=off", "-x", "c++",
          "-I", CSRC, "-I", GEN, os.path.join(CSRC, "host_emulator.cpp"), "-o", tmp], verbose)
    os.replace(tmp, EMU)
    return EMU


def build(force=False, verbose=False, emulator=True) -> None:
    build_lib(force=force, verbose=verbose)
    if emulator:
        build_emulator(force=force, verbose=verbose)


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--no-emulator", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print -Xptxas -v register/spill report")
    ap.add_argument("-v", "--verbose", action="store_true")
    a = ap.parse_args(argv)
    build_lib(force=a.force or a.ptxas_info, verbose=a.verbose, ptxas_info=a.ptxas_info)
    if not a.no_emulator:
        build_emulator(force=a.force, verbose=a.verbose)
    print(LIB)
    return 0


if __name__ == "__main__":
    sys.exit(main())
