"""Build the CUDA library ``libfa.so`` in-tree (sm_100a only).

``python -m exact_io_aware_51_b200.build`` compiles every ``csrc/*.cu`` with
nvcc for ``sm_100a``: the product library ``exact_io_aware_51_b200/libfa.so``;
the checking build ``libfa_debug.so`` (the same sources with ``FA_DEBUG``:
device-side bounds checks that record a status and skip the access); and, from
``fa_probe.cu`` alone, the test library ``libfa_probe.so`` (single MMA tile
probes; declared in ``csrc/fa_testing.h``, not in the public header).
nvcc cross-compiles without a GPU.  The CUDA runtime is linked statically, so
the libraries only need the driver at run time.
"""

from __future__ import annotations

import concurrent.futures
import os
import pathlib
import shutil
import subprocess
import sys

PKG = pathlib.Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
INCLUDE = ROOT / "include"
BUILD = PKG / "_build"
LIB = PKG / "libfa.so"
SOURCES = ("fa_api.cu", "fa_fwd_bf16.cu", "fa_fwd_fp8.cu", "fa_fwd_f32.cu", "fa_bwd.cu",
           "fa_bwd_static.cu", "fa_ring.cu",
           "fa_bwd64.cu", "fa_decode.cu")
PROBE_SOURCES = ("fa_probe.cu",)
PROBE_LIB = PKG / "libfa_probe.so"
DEBUG_LIB = PKG / "libfa_debug.so"
ARCH = ("-gencode", "arch=compute_100a,code=sm_100a")
FLAGS = ("-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr")


def nvcc() -> str:
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libfa.so")
    return exe


def _deps():
    return ([CSRC / s for s in SOURCES + PROBE_SOURCES] + list(CSRC.glob("*.cuh")) + list(CSRC.glob("*.h"))
            + [INCLUDE / "fa.h", pathlib.Path(__file__)])


def up_to_date() -> bool:
    libs = (LIB, PROBE_LIB, DEBUG_LIB)
    if not all(p.exists() for p in libs):
        return False
    t = min(p.stat().st_mtime for p in libs)
    return all(p.stat().st_mtime <= t for p in _deps())


def _compile(src: pathlib.Path, verbose: bool, debug: bool = False) -> pathlib.Path:
    obj = BUILD / (src.stem + ("_debug.o" if debug else ".o"))
    cmd = [nvcc(), *ARCH, *FLAGS, *(("-DFA_DEBUG",) if debug else ()), "-I", str(INCLUDE), "-I", str(CSRC), "-c",
           str(src), "-o", str(obj)]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src.name}:\n{r.stdout}\n{r.stderr}")
    if verbose and r.stderr:
        print(r.stderr, flush=True)
    return obj


def build(force: bool = False, verbose: bool = False) -> pathlib.Path:
    """Compile and link libfa.so unless it is newer than every source."""
    if not force and up_to_date():
        return LIB
    BUILD.mkdir(exist_ok=True)
    jobs = [(s, False) for s in SOURCES + PROBE_SOURCES] + [(s, True) for s in SOURCES]
    with concurrent.futures.ThreadPoolExecutor(max_workers=len(jobs)) as ex:
        objs = dict(zip(jobs, ex.map(lambda j: _compile(CSRC / j[0], verbose, j[1]), jobs)))
    for lib, srcs, debug in ((LIB, SOURCES, False), (PROBE_LIB, PROBE_SOURCES, False), (DEBUG_LIB, SOURCES, True)):
        tmp = lib.with_suffix(".so.tmp")
        cmd = [nvcc(), *ARCH, "-shared", "-o", str(tmp), *(str(objs[(s, debug)]) for s in srcs), "-cudart", "static"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link of {lib.name} failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib)
    return LIB


if __name__ == "__main__":
    p = build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(p)
