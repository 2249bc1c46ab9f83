"""Build libbbc.so (the C-ABI library) in-tree for sm_100a.

Each source is compiled by nvcc (no relocatable device code: every kernel and
its launcher share a translation unit), then linked into one shared library
next to this file. `python -m blockwise_bit_codebook_b200.build [--force] [--debug]`.
--debug builds libbbc_debug.so instead: the same sources with -DBBC_DEBUG, whose
kernels check every computed global address against its buffer's extent and
report failures through bbc_debug_status (load it with BBC_LIBRARY=...).
"""
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.environ.get("BBC_BUILD_OUTPUT") or os.path.join(HERE, "libbbc.so")
LIB_DEBUG = os.path.join(HERE, "libbbc_debug.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "-I", INCLUDE, "-I", CSRC]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) \
        + [os.path.join(INCLUDE, "bbc.h"), __file__]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra=(), debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if debug:
        extra = (*extra, "-DBBC_DEBUG")
    if not force and not _stale(lib):
        return lib
    tmp = tempfile.mkdtemp(prefix="bbc_build_")
    try:
        def compile_one(src):
            obj = os.path.join(tmp, os.path.basename(src) + ".o")
            cmd = [NVCC, *ARCH, *FLAGS, *os.environ.get("BBC_NVCC_EXTRA", "").split(), *extra,
                   "-c", src, "-o", obj]
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0 or verbose:
                sys.stderr.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
            if r.returncode != 0:
                raise RuntimeError(f"nvcc failed on {src}")
            return obj
        with cf.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
            objs = list(ex.map(compile_one, sources()))
        out = os.path.join(tmp, "libbbc.so")
        cmd = [NVCC, *ARCH, "-shared", "-o", out, *objs]
        subprocess.run(cmd, check=True)
        shutil.move(out, lib)
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
    return lib


if __name__ == "__main__":
    extra = ["-Xptxas", "-v"] if "--ptxas" in sys.argv else []
    print(build(force="--force" in sys.argv or bool(extra), verbose="-v" in sys.argv or bool(extra), extra=extra,
                debug="--debug" in sys.argv))
