"""Build the sm_100a shared library libhyena_b200.so in-tree.

    python -m fft_long_convolution_implicit_b200.build [--force] [--verbose-ptxas] [--tc05]

--tc05 builds the variant whose bf16, L = 2048 forward runs on the tcgen05
kernel (csrc/tc05.cu) instead of the mma.sync one (-DHYENA_TC05=1); the
choice is remembered in lib/build_options.txt; build() called without a
variant (as the tests and bench.py do) keeps the recorded one, and
`python -m ...build` without --tc05 builds the default.

Each csrc/*.cu is compiled separately (in parallel) with
``-gencode arch=compute_100a,code=sm_100a -lineinfo`` and linked into
fft_long_convolution_implicit_b200/lib/libhyena_b200.so. nvcc cross-compiles,
so no GPU is needed to build.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJ = os.path.join(PKG, "_build")
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libhyena_b200.so")
OPTIONS = os.path.join(LIBDIR, "build_options.txt")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu*")) + glob.glob(os.path.join(CSRC, "*.h"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def _defines(tc05: bool) -> list[str]:
    return ["-DHYENA_TC05=1"] if tc05 else []


def up_to_date(tc05: bool = False) -> bool:
    if not os.path.exists(LIB) or not os.path.exists(OPTIONS):
        return False
    with open(OPTIONS) as f:
        if f.read().strip() != " ".join(_defines(tc05)):
            return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in _deps() + [__file__])


def built_tc05() -> bool:
    """The variant recorded by the last build (False when none is recorded)."""
    try:
        with open(OPTIONS) as f:
            return "HYENA_TC05=1" in f.read()
    except OSError:
        return False


def build(force: bool = False, verbose_ptxas: bool = False, quiet: bool = True, tc05: bool | None = None) -> str:
    """tc05=None keeps the variant of the last build (the default one if none)."""
    if tc05 is None:
        tc05 = built_tc05()
    if not force and up_to_date(tc05):
        return LIB
    os.makedirs(OBJ, exist_ok=True)
    os.makedirs(LIBDIR, exist_ok=True)
    cc = nvcc()
    srcs = _sources()

    def compile_one(src):
        obj = os.path.join(OBJ, os.path.basename(src) + ".o")
        cmd = [cc, *ARCH, *FLAGS, *_defines(tc05), "-c", src, "-o", obj]
        if verbose_ptxas:
            cmd += ["-Xptxas", "-v"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        return obj, r.stdout + r.stderr

    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(compile_one, srcs))
    if verbose_ptxas:
        for _, log in results:
            sys.stdout.write(log)
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [cc, *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", tmp, *[o for o, _ in results]]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    with open(OPTIONS, "w") as f:
        f.write(" ".join(_defines(tc05)) + "\n")
    if not quiet:
        print(f"built {LIB}")
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--tc05", action="store_true", help="bf16 L=2048 forward on the tcgen05 kernel")
    a = ap.parse_args()
    build(force=a.force, verbose_ptxas=a.verbose_ptxas, quiet=False, tc05=bool(a.tc05))
