"""Build ``libcider.so`` (the C-ABI library) in-tree with nvcc for sm_100a.

Every translation unit under ``csrc/`` is compiled with
``-gencode arch=compute_100a,code=sm_100a -O3 -lineinfo`` (no fast-math:
the activation quantization relies on IEEE division) and linked into one
shared library next to this file.  The build is incremental: a unit is
recompiled when it or any header under ``csrc/`` or ``include/`` is newer
than its object.
"""
import glob
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
INCLUDE = os.path.join(ROOT, "include")
OBJDIR = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libcider.so")

NVCC = os.environ.get("NVCC", "nvcc")
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    f"-I{INCLUDE}",
]


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _compile(src, extra):
    obj = os.path.join(OBJDIR, os.path.basename(src) + ".o")
    newest = max([os.path.getmtime(src)] + [os.path.getmtime(h) for h in _headers()])
    if os.path.exists(obj) and os.path.getmtime(obj) >= newest:
        return obj
    cmd = [NVCC, *NVCC_FLAGS, *extra, "-c", src, "-o", obj + ".tmp"]
    subprocess.run(cmd, check=True)
    os.replace(obj + ".tmp", obj)
    return obj


def build_library(verbose_ptxas: bool = False) -> str:
    """Compile every ``csrc/*.cu`` and link ``libcider.so``; returns its path."""
    os.makedirs(OBJDIR, exist_ok=True)
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    with ThreadPoolExecutor(max_workers=max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra), srcs))
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(o) for o in objs):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.run([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-o", tmp, *objs, "-lcudart"], check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    import sys
    print(build_library(verbose_ptxas="-v" in sys.argv))
