"""Build of the in-tree C-ABI library ``lib/libsi.so`` for sm_100a.

``python -m streaming_top_indexer_b200.build`` compiles every CUDA source of
the package with nvcc (no GPU needed) into a shared library that exports the
functions declared in ``include/si.h``.
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_DIR = os.path.join(PKG, "lib")
LIB_PATH = os.path.join(LIB_DIR, "libsi.so")
TRACE_LIB_PATH = os.path.join(LIB_DIR, "libsi_trace.so")  # cycle-tracing build (SI_TRACE)
# Test-only build (SI_FAULT_TEST) whose select kernel withholds one signal so
# that a bounded device wait expires; used by the abort-path GPU test only.
FAULT_TEST_LIB_PATH = os.path.join(LIB_DIR, "libsi_ftest.so")
# Timeline-tracing variant of the sparse attention kernel (SI_ATTN_TRACE).
ATTN_TRACE_LIB_PATH = os.path.join(LIB_DIR, "libsi_atrace.so")
# The host library, one translation unit per H_I of the select kernel and the
# sparse attention stage, compiled in parallel and linked into one library.
SOURCES = [os.path.join(CSRC, f) for f in ("si_lib.cu", "si_select_h8.cu", "si_select_h16.cu", "si_select_h32.cu",
                                           "si_select_h64.cu", "si_attn.cu", "si_proj.cu", "si_host_io.cu")]
BUILD_DIR = os.path.join(PKG, "_build")
HEADERS = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + [
    os.path.join(INCLUDE, "si.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-cudart=shared",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def needs_build(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS)


def build_fault_test(force: bool = False, verbose: bool = False) -> str:
    """The SI_FAULT_TEST variant, lib/libsi_ftest.so (abort-path test only)."""
    if not force and not needs_build(FAULT_TEST_LIB_PATH):
        return FAULT_TEST_LIB_PATH
    return build(verbose=verbose, extra=["-DSI_FAULT_TEST"], out=FAULT_TEST_LIB_PATH)


def _compile(src: str, obj: str, extra, verbose: bool) -> None:
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed on {os.path.basename(src)} ({res.returncode}):\n{res.stderr[-8000:]}")
    if verbose and res.stderr:
        print(res.stderr, file=sys.stderr)


def build(force: bool = False, verbose: bool = False, extra=(), trace: bool = False, out: str | None = None) -> str:
    """Compile every CUDA source (in parallel) and link ``lib/libsi.so``.

    ``trace`` builds the cycle-tracing variant (SI_TRACE) into
    ``lib/libsi_trace.so``; ``out`` names another output for a variant built
    with ``extra`` flags."""
    if out is None:
        out = TRACE_LIB_PATH if trace else LIB_PATH
    if out == LIB_PATH and not extra and not force and not needs_build():
        return LIB_PATH
    os.makedirs(LIB_DIR, exist_ok=True)
    tag = os.path.splitext(os.path.basename(out))[0]
    obj_dir = os.path.join(BUILD_DIR, tag)
    os.makedirs(obj_dir, exist_ok=True)
    if trace:
        extra = [*extra, "-DSI_TRACE"]
    objs = [os.path.join(obj_dir, os.path.splitext(os.path.basename(f))[0] + ".o") for f in SOURCES]
    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        for f in [ex.submit(_compile, src, obj, list(extra), verbose) for src, obj in zip(SOURCES, objs)]:
            f.result()
    tmp = out + ".tmp"
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-cudart=shared", "-shared", *objs, "-o", tmp,
           "-Xlinker", "-rpath,/usr/local/cuda/lib64"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc link failed ({res.returncode}):\n{res.stderr[-8000:]}")
    os.replace(tmp, out)
    return out


CUT_BENCH_SRC = os.path.join(CSRC, "si_cut_bench.cu")
CUT_BENCH_PATH = os.path.join(BUILD_DIR, "si_cut_bench")  # microbenchmark of the pool cut (development tool)


def build_cut_bench(verbose: bool = False) -> str:
    """The pool-cut microbenchmark executable (not part of the library)."""
    os.makedirs(BUILD_DIR, exist_ok=True)
    cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, CUT_BENCH_SRC, "-o", CUT_BENCH_PATH]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed on si_cut_bench.cu ({res.returncode}):\n{res.stderr[-8000:]}")
    return CUT_BENCH_PATH


if __name__ == "__main__":
    if "--cut-bench" in sys.argv:
        print(build_cut_bench(verbose=True))
    elif "--attn-trace" in sys.argv:
        print(build(verbose=True, extra=["-DSI_ATTN_TRACE"], out=ATTN_TRACE_LIB_PATH))
    elif "--fault-test" in sys.argv:
        print(build_fault_test(force=True, verbose=True))
    else:
        print(build(force="--force" in sys.argv, verbose=True, trace="--trace" in sys.argv,
                    extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []))
