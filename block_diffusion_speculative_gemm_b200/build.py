"""Builds libdflash.so (every CUDA source under csrc/) for sm_100a with nvcc.

Usage: ``python -m block_diffusion_speculative_gemm_b200.build`` (or call
``build()``).  The library lands next to this file so it travels with the
source tree.  Rebuilds only when a source is newer than the library.
"""

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libdflash.so")
# the same sources with DFLASH_CHECKED: index checks that set DFLASH_DEV_CHECK
# and skip the access, for test runs (the stand-in for a memory checker)
LIB_CHECKED = os.path.join(HERE, "libdflash_checked.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-Xptxas", "-warn-spills",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    deps += glob.glob(os.path.join(INCLUDE, "*.h")) + [__file__]
    return any(os.path.getmtime(p) > t for p in deps)


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed: " + " ".join(cmd[-3:]))
    if verbose and (r.stdout or r.stderr):
        sys.stderr.write(r.stdout + r.stderr)


def build(force: bool = False, verbose: bool = False, extra=(), checked: bool = False) -> str:
    """Compiles every source to an object in parallel under _build/, then links."""
    from concurrent.futures import ThreadPoolExecutor

    lib = LIB_CHECKED if checked else LIB
    if not force and not _stale(lib):
        return lib
    flags = [*NVCC_FLAGS, *(["-DDFLASH_CHECKED"] if checked else []), *extra]
    objdir = os.path.join(os.path.dirname(HERE), "_build", "checked" if checked else "release")
    os.makedirs(objdir, exist_ok=True)
    objs = [os.path.join(objdir, os.path.basename(src)[:-3] + ".o") for src in sources()]
    compile_flags = [f for f in flags if f != "-shared"]
    with ThreadPoolExecutor(max_workers=max(1, min(len(objs), os.cpu_count() or 4))) as ex:
        list(ex.map(lambda so: _run([_nvcc(), *compile_flags, "-I", INCLUDE, "-c", "-o", so[1],
                                     so[0]], verbose), zip(sources(), objs)))
    tmp = lib + ".tmp"
    _run([_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-Xcompiler", "-fPIC",
          "-o", tmp, *objs], verbose)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=("-Xptxas", "-v") if "--ptxas-v" in sys.argv else (),
          checked="--checked" in sys.argv)
