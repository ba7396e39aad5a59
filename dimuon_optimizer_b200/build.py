"""Builds libdimuon.so in-tree with nvcc for sm_100a.

    python dimuon_optimizer_b200/build.py [--debug]

The library is compiled for B200 only (-gencode arch=compute_100a,code=sm_100a)
and links the CUDA runtime statically; the driver's tensor-map encoder is
looked up at run time, so no -lcuda is needed.
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libdimuon.so")
SOURCES = ["api.cu", "api_noalloc.cu", "k_elementwise.cu", "k_ns_simt.cu", "k_ns_tc.cu", "k_ns_tc2.cu", "k_thin.cu", "k_thin_bulk.cu", "k_thin_cluster.cu"]
HEADERS = ["dm_common.cuh", "dm_internal.h", "dm_sm100.cuh", "dm_tiles.cuh", "dm_tc_epilogue.cuh", "dm_thin.cuh"]


def nvcc_path():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [
        os.path.join(INCLUDE, "dimuon.h"), os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force=False, verbose=False, extra=()):
    """Compiles each source to an object in parallel (objects under a
    temporary folder), then links the shared library."""
    if not force and not _stale():
        return LIB
    import tempfile
    from concurrent.futures import ThreadPoolExecutor

    flags = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
             "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]
    flags += list(extra)
    with tempfile.TemporaryDirectory(prefix="dimuon_build_") as tmp:
        def compile_one(src):
            obj = os.path.join(tmp, src.replace(".cu", ".o"))
            cmd = [nvcc_path()] + flags + ["-c", os.path.join(CSRC, src), "-o", obj]
            if verbose:
                print(" ".join(cmd), flush=True)
            subprocess.run(cmd, check=True)
            return obj

        workers = max(1, min(len(SOURCES), os.cpu_count() or 1))
        with ThreadPoolExecutor(max_workers=workers) as pool:
            objs = list(pool.map(compile_one, SOURCES))
        link = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                "-Xcompiler", "-fPIC", "-o", LIB + ".tmp"] + objs
        if verbose:
            print(" ".join(link), flush=True)
        subprocess.run(link, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose=True, extra=["-Xptxas", "-v"] if "-v" in sys.argv else [])
