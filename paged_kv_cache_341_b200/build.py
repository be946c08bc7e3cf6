"""Build ``libpagedattn.so`` in-tree for sm_100a (nvcc + g++, no GPU needed).

``python -m paged_kv_cache_341_b200.build`` compiles
``csrc/pa_device.cu`` (all kernels) and the host pool into
``paged_kv_cache_341_b200/libpagedattn.so``.  The CUDA runtime is linked
statically; the driver's ``cuTensorMapEncodeTiled`` is looked up at run time,
so the library has no link-time dependency on libcuda.
"""

import hashlib
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libpagedattn.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xptxas", "-v"]
CXX_FLAGS = ["-O2", "-std=c++17", "-fPIC", "-Wall"]
SOURCES_CU = ["pa_device.cu"]
SOURCES_CPP = ["pool.cpp", "prefix_cache.cpp", "common.cpp", "engine.cpp"]
CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _inputs_digest():
    h = hashlib.sha256()
    files = sorted(os.listdir(CSRC)) + ["../../include/pa.h"]
    for name in files:
        path = os.path.normpath(os.path.join(CSRC, name))
        if os.path.isfile(path):
            h.update(name.encode())
            with open(path, "rb") as f:
                h.update(f.read())
    h.update(" ".join(ARCH + NVCC_FLAGS + CXX_FLAGS).encode())
    return h.hexdigest()


def _run(cmd, log):
    res = subprocess.run(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
    log.append("$ " + " ".join(cmd) + "\n" + res.stdout)
    if res.returncode != 0:
        raise RuntimeError("build step failed:\n" + log[-1])


def build(verbose=False):
    """Compile and link; returns the library path.  Writes the ptxas report to _build/ptxas.txt."""
    os.makedirs(BUILD, exist_ok=True)
    log = []
    objs = []
    for src in SOURCES_CU:
        obj = os.path.join(BUILD, src + ".o")
        _run([nvcc()] + ARCH + NVCC_FLAGS + ["-I", INCLUDE, "-I", CSRC, "-c", os.path.join(CSRC, src), "-o", obj], log)
        objs.append(obj)
    for src in SOURCES_CPP:
        obj = os.path.join(BUILD, src + ".o")
        _run(["g++"] + CXX_FLAGS + ["-I", INCLUDE, "-I", CSRC, "-I", os.path.join(CUDA_HOME, "include"), "-c",
                                   os.path.join(CSRC, src), "-o", obj], log)
        objs.append(obj)
    tmp = LIB + ".tmp"
    _run([nvcc()] + ARCH + ["-shared", "-o", tmp] + objs, log)
    os.replace(tmp, LIB)
    with open(os.path.join(BUILD, "ptxas.txt"), "w") as f:
        f.write("\n".join(log))
    with open(os.path.join(BUILD, "digest.txt"), "w") as f:
        f.write(_inputs_digest())
    if verbose:
        print("\n".join(log))
    return LIB


def kernel_digest():
    """Digest of the decode kernel's sources and launch code (ties ncu counters to the code they were taken on)."""
    h = hashlib.sha256()
    for name in ("decode.cuh", "ptx.cuh", "dtype.cuh", "launch_decode.cuh"):
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def up_to_date():
    try:
        with open(os.path.join(BUILD, "digest.txt")) as f:
            return os.path.exists(LIB) and f.read().strip() == _inputs_digest()
    except OSError:
        return False


def ensure_built():
    """Build when the library is missing, its sources changed, or its build record is missing.

    A library without ``_build/digest.txt`` beside it cannot be tied to the
    sources in the tree, so it is rebuilt rather than trusted; if that build
    fails, the error says so instead of loading a library of unknown origin.
    Returns the path."""
    if up_to_date():
        return LIB
    try:
        return build()
    except (OSError, RuntimeError) as e:
        raise RuntimeError("libpagedattn.so is missing or does not match its sources (no build record, or "
                           "a different digest), and rebuilding it failed: %s" % e) from e


if __name__ == "__main__":
    build(verbose="-v" in sys.argv)
    print(LIB)
