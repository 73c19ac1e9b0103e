"""Build the CUDA library ``libfa.so`` in-tree (sm_100a only).

``python -m exact_io_aware_51_b200.build`` compiles every ``csrc/*.cu`` with
nvcc for ``sm_100a``: the product library ``exact_io_aware_51_b200/libfa.so``
and, from ``fa_probe.cu`` alone, the test library ``libfa_probe.so`` (single
MMA tile probes; declared in ``csrc/fa_testing.h``, not in the public header).
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
    if not LIB.exists() or not PROBE_LIB.exists():
        return False
    t = min(LIB.stat().st_mtime, PROBE_LIB.stat().st_mtime)
    return all(p.stat().st_mtime <= t for p in _deps())


def _compile(src: pathlib.Path, verbose: bool) -> pathlib.Path:
    obj = BUILD / (src.stem + ".o")
    cmd = [nvcc(), *ARCH, *FLAGS, "-I", str(INCLUDE), "-I", str(CSRC), "-c", str(src), "-o", str(obj)]
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
    every = SOURCES + PROBE_SOURCES
    with concurrent.futures.ThreadPoolExecutor(max_workers=len(every)) as ex:
        objs = dict(zip(every, ex.map(lambda s: _compile(CSRC / s, verbose), every)))
    for lib, srcs in ((LIB, SOURCES), (PROBE_LIB, PROBE_SOURCES)):
        tmp = lib.with_suffix(".so.tmp")
        cmd = [nvcc(), *ARCH, "-shared", "-o", str(tmp), *(str(objs[s]) for s in srcs), "-cudart", "static"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link of {lib.name} failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib)
    return LIB


if __name__ == "__main__":
    p = build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(p)
