"""Builds libfa.so (the C-ABI attention library) in-tree with nvcc for sm_100a.

    python -m exact_attention_107_b200.build [--force] [--verbose]

The shared library links the CUDA runtime statically and resolves the one
driver entry point it needs (cuTensorMapEncodeTiled) at run time, so it loads
on a machine without a GPU driver; calls then fail with FA_ERR_CUDA.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import pathlib
import subprocess
import sys

PKG = pathlib.Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
INCLUDE = ROOT / "include"
BUILD = PKG / "_build"
LIB = PKG / "libfa.so"
# Test-only build: every pipeline wait limited to 100 clocks (far less than any tile load
# takes), so that each kernel runs a wait out and takes its error path.
TIMEOUT_TEST_LIB = PKG / "libfa_timeout_test.so"
# Debug build: device-side bounds checks of computed indices and warp-convergence checks at
# the warp-collective tensor-memory phases (a failed check records FA_ERR_DEBUG_CHECK).
DEBUG_LIB = PKG / "libfa_debug.so"
VARIANTS = {"timeout_test": ["-DFA_WAIT_LIMIT_CYCLES=100"], "debug": ["-DFA_DEBUG_CHECKS"]}
SOURCES = ["fa_api.cu", "fa_fwd_sm100.cu", "fa_fwd_d256_sm100.cu", "fa_fwd_f32.cu", "fa_bwd_sm100.cu",
           "fa_bwd_d256_sm100.cu", "fa_bwd_fused_sm100.cu", "fa_noalloc.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC",
          "-I" + str(INCLUDE), "-I" + str(CSRC)]


def nvcc() -> str:
    cand = os.environ.get("NVCC") or "/usr/local/cuda/bin/nvcc"
    return cand if os.path.exists(cand) else "nvcc"


def _deps():
    return ([CSRC / s for s in SOURCES] + list(CSRC.glob("*.cuh")) + list(CSRC.glob("*.h")) + [INCLUDE / "fa.h"]
            + [pathlib.Path(__file__).resolve()])


def up_to_date() -> bool:
    libs = (LIB, TIMEOUT_TEST_LIB, DEBUG_LIB)
    if not all(lib.exists() for lib in libs):
        return False
    t = min(lib.stat().st_mtime for lib in libs)
    return all(p.stat().st_mtime <= t for p in _deps())


def _compile(src: str, verbose: bool, ptxas_v: bool, variant: str = "") -> pathlib.Path:
    out = BUILD / variant if variant else BUILD
    out.mkdir(parents=True, exist_ok=True)
    obj = out / (pathlib.Path(src).stem + ".o")
    cmd = [nvcc(), *ARCH, *CFLAGS, *VARIANTS.get(variant, []), "-c", str(CSRC / src), "-o", str(obj)]
    if ptxas_v:
        cmd += ["-Xptxas", "-v"]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if ptxas_v or verbose:
        sys.stdout.write(r.stderr)
    return obj


def _link(objs, lib: pathlib.Path, verbose: bool) -> None:
    tmp = lib.with_suffix(".so.tmp")
    cmd = [nvcc(), *ARCH, "-shared", "-o", str(tmp), *map(str, objs), "-cudart", "static"]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False, ptxas_v: bool = False) -> pathlib.Path:
    """Compiles every CUDA source for sm_100a and links libfa.so next to this file, the
    test-only libfa_timeout_test.so (the same sources with short pipeline-wait limits) and
    libfa_debug.so (the same sources with device-side bounds and convergence checks)."""
    if not force and not ptxas_v and up_to_date():
        return LIB
    BUILD.mkdir(exist_ok=True)
    jobs = [(s, v) for v in ("", "timeout_test", "debug") for s in SOURCES]
    with cf.ThreadPoolExecutor(max_workers=min(len(jobs), max(4, os.cpu_count() or 4))) as ex:
        objs = list(ex.map(lambda j: _compile(j[0], verbose, ptxas_v and not j[1], j[1]), jobs))
    n = len(SOURCES)
    _link(objs[:n], LIB, verbose)
    _link(objs[n:2 * n], TIMEOUT_TEST_LIB, verbose)
    _link(objs[2 * n:], DEBUG_LIB, verbose)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true", help="print registers / spills per kernel")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, ptxas_v=a.ptxas_v))
