"""Build ``libcowa.so`` (the CoWA C-ABI library) in-tree for sm_100a.

Each ``csrc/*.cu`` is compiled by nvcc for ``arch=compute_100a,code=sm_100a``
into ``_build/`` and linked into a shared library next to this file, so the
binary travels with the source tree.  Run ``python -m
structured_sparse_attention_block_b200.build`` or call ``build()``.

``build(debug=True)`` (``--debug``) builds the checking variant
``libcowa_debug.so`` from the same sources with ``-DCOWA_DEBUG`` (objects in
``_build_debug/``): its kernels check tile, row and workspace indices against
the extents they must stay within and report a failed check as
COWA_ERR_DEVICE instead of making the access.  The binding loads it instead
of ``libcowa.so`` when the environment sets ``COWA_DEBUG=1``.
"""
import concurrent.futures
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libcowa.so")
OUT_DEBUG = os.path.join(HERE, "_build_debug")
LIB_DEBUG = os.path.join(HERE, "libcowa_debug.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    "-I", INCLUDE,
]


def _nvcc():
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    path = os.path.join(cuda, "bin", "nvcc")
    return path if os.path.exists(path) else "nvcc"


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _deps():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(INCLUDE, "cowa.h"))
    files.append(os.path.abspath(__file__))
    return files


def _compile(src, extra, verbose, out=OUT):
    obj = os.path.join(out, os.path.basename(src)[:-3] + ".o")
    cmd = [_nvcc(), *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed for %s:\n%s\n%s" % (src, res.stdout, res.stderr))
    return obj, res.stderr


def build(force: bool = False, verbose: bool = False, extra=(), debug: bool = False) -> str:
    """Compile every kernel source and link ``libcowa.so`` (``debug``: the
    checking variant ``libcowa_debug.so``); return its path."""
    lib, out = (LIB_DEBUG, OUT_DEBUG) if debug else (LIB, OUT)
    extra = list(extra) + (["-DCOWA_DEBUG"] if debug else [])
    if not force and os.path.exists(lib):
        newest = max(os.path.getmtime(f) for f in _deps())
        if os.path.getmtime(lib) >= newest:
            return lib
    os.makedirs(out, exist_ok=True)
    with concurrent.futures.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        results = list(ex.map(lambda s: _compile(s, extra, verbose, out), sources()))
    if verbose:
        for _, log in results:
            sys.stderr.write(log)
    tmp = lib + ".tmp.%d" % os.getpid()
    cmd = [_nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
           "-o", tmp, *[o for o, _ in results], "-lcudart"]
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
