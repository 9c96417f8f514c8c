"""Build libquarot.so in-tree with nvcc for sm_100a (B200).

One translation unit (csrc/quarot_api.cu) includes every kernel header, so the
device-side status word is a single symbol.  The CUDA runtime is linked
statically; the library needs only the NVIDIA driver at run time.
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libquarot.so")
# the bounds-checking build: every kernel checks its output stores
# (QUAROT_DEBUG_BOUNDS; see quarot_debug_bounds in include/quarot.h)
LIB_DEBUG = os.path.join(PKG, "libquarot_dbg.so")
SOURCES = [os.path.join(CSRC, "quarot_api.cu")]
HEADERS = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + \
    [os.path.join(ROOT, "include", "quarot.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
    "--expt-relaxed-constexpr",
]


def _nvcc():
    home = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    p = os.path.join(home, "bin", "nvcc")
    return p if os.path.exists(p) else "nvcc"


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False, debug_bounds: bool = False) -> str:
    lib = LIB_DEBUG if debug_bounds else LIB
    if not force and up_to_date(lib):
        return lib
    cmd = [_nvcc()] + NVCC_FLAGS + ["-I", os.path.join(ROOT, "include"), "-I", CSRC]
    if debug_bounds:
        cmd += ["-DQUAROT_DEBUG_BOUNDS"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += ["-o", lib + ".tmp"] + SOURCES
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


def build_all(force: bool = False) -> None:
    """The normal library and the bounds-checking one, compiled side by side."""
    import concurrent.futures as cf
    with cf.ThreadPoolExecutor(2) as ex:
        for f in [ex.submit(build, force, False, False), ex.submit(build, force, False, True)]:
            f.result()


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv, debug_bounds="--debug-bounds" in sys.argv))
