"""Build librownorm.so (the C-ABI CUDA library) in-tree for sm_100a.

The kernel instantiation tables are generated into the build directory
(csrc/gen_instantiations.py), each translation unit compiles in its own nvcc
process (the tables are independent), then everything links into one shared library
with the CUDA runtime linked statically and only the ``rn_*`` entry points of
``include/rownorm.h`` exported.
"""
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "librownorm.so")

# hand-written translation units; the kernel instantiation tables are
# generated into the build directory by csrc/gen_instantiations.py
SOURCES = ["rownorm_api.cu", "rownorm_stream.cu"]
HEADERS = ["rownorm_core.cuh", "rownorm_kernels.cuh", "rownorm_ring.cuh", "rownorm_launch.h",
           "rownorm_stream.cuh", "gen_instantiations.py"]
GEN = os.path.join(BUILD, "gen")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                 "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build librownorm.so")
    return path


def _newest_input() -> float:
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "rownorm.h"))
    files.append(os.path.abspath(__file__))
    return max(os.path.getmtime(f) for f in files)


def _compile(src: str, extra) -> str:
    obj = os.path.join(BUILD, os.path.splitext(os.path.basename(src))[0] + ".o")
    path = src if os.path.isabs(src) else os.path.join(CSRC, src)
    cmd = [nvcc()] + CFLAGS + list(extra) + ["-c", path, "-o", obj]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{res.stdout}\n{res.stderr}")
    return obj, res.stderr


def build(force: bool = False, verbose_ptxas: bool = False, jobs: int = 0) -> str:
    """Compile and link; returns the library path. Skips work when the
    library is newer than every source."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= _newest_input():
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    sys.path.insert(0, CSRC)
    try:
        import gen_instantiations
    finally:
        sys.path.remove(CSRC)
    units = SOURCES + gen_instantiations.write_tables(GEN)
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    jobs = jobs or min(len(units), os.cpu_count() or 1)
    with cf.ThreadPoolExecutor(jobs) as ex:
        results = list(ex.map(lambda s: _compile(s, extra), units))
    if verbose_ptxas:
        for _, log in results:
            sys.stderr.write(log)
    objs = [o for o, _ in results]
    tmp = LIB + ".tmp"
    cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs + [
        "-Xlinker", "--exclude-libs,ALL", "-lrt", "-ldl", "-lpthread"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"link failed:\n{res.stdout}\n{res.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
