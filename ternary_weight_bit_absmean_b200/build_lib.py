"""Build ``libbitlinear.so`` (the CUDA kernels and the C ABI) in-tree for sm_100a.

``python -m ternary_weight_bit_absmean_b200.build_lib [--force] [--verbose] [--debug]``

``--debug`` builds ``libbitlinear_debug.so`` instead: the same library with the device
index checks on (``BL_DEBUG_CHECKS=1``; a failed check ORs ``BL_ERRBIT_INDEX`` into the
caller's error word and skips the access), for debugging without a sanitizer.

The library is compiled with nvcc for ``sm_100a`` only, position independent, with the
CUDA runtime linked statically (no dependency on the runtime that PyTorch ships) and
without linking the driver library (the tensor-map encoder is fetched through the
runtime's driver entry point), so it loads on a machine without a GPU.
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libbitlinear.so")
DEBUG_LIB = os.path.join(PKG, "libbitlinear_debug.so")
SOURCES = ["bl_api.cu", "k_quant.cu", "k_gemv.cu", "k_gemv_tma.cu", "k_gemv_tc.cu", "k_gemv_stream.cu", "k_gemm_tc.cu", "k_gemm_tc2.cu", "bl_noalloc.cu", "k_tl5.cu", "k_ste.cu"]
HEADERS = ["bl_device.cuh", "bl_internal.h"]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-cudart", "static"]


def _inputs():
    return ([os.path.join(CSRC, f) for f in SOURCES + HEADERS]
            + [os.path.join(INCLUDE, "bitlinear.h"), os.path.abspath(__file__)])


def source_digest(files=None) -> str:
    """SHA-256 over the library's sources and header (identifies a kernel build), or
    over the given source files only (identifies the kernels they define)."""
    import hashlib
    h = hashlib.sha256()
    paths = ([os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "bitlinear.h")]
             if files is None else [os.path.join(CSRC, f) for f in files])
    for p in paths:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# The files that define the prefill kernels (their device code and the helpers it
# inlines): DRAM counters taken on these kernels stay valid while these are unchanged.
PREFILL_KERNEL_FILES = ["k_gemm_tc.cu", "k_gemm_tc2.cu", "bl_device.cuh"]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = DEBUG_LIB if debug else LIB
    if not force and up_to_date(lib):
        return lib
    objdir = os.path.join(PKG, "_build_debug" if debug else "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    for src in SOURCES:
        obj = os.path.join(objdir, src.replace(".cu", ".o"))
        cmd = [NVCC, *FLAGS, *(["-DBL_DEBUG_CHECKS=1"] if debug else []), "-I", INCLUDE, "-I", CSRC, "-c",
               os.path.join(CSRC, src), "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = lib + ".tmp.%d" % os.getpid()
    subprocess.run([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-cudart", "static",
                    *objs, "-o", tmp], check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, debug="--debug" in sys.argv))
