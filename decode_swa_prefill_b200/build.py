"""Build libswa.so in-tree with nvcc for sm_100a (cross-compiles; no GPU needed).

    python -m decode_swa_prefill_b200.build [--verbose-ptxas] [--debug]

--debug builds libswa_debug.so instead: the same kernels compiled with
-DSWA_DEBUG, whose device-side checks of tile, row and slot indices record
SWA_ERR_INTERNAL in the status word (loaded when SWA_DEBUG=1 is set).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libswa.so")
DEBUG_LIB = os.path.join(HERE, "libswa_debug.so")
SOURCES = ["swa_abi.cu", "prefill_tc.cu", "prefill_pp.cu", "narrow_tc.cu", "simt_kernels.cu", "decode_noalloc.cu",
           "dilated.cu", "backward_tc.cu"]
HEADERS = ["ptx.cuh", "swa_internal.h", "tma_map.h"]


def nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _stale(lib):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "swa.h")]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force=False, ptxas_verbose=False, debug=False):
    lib = DEBUG_LIB if debug else LIB
    if not force and not _stale(lib):
        return lib
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [nvcc(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
           "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE, "-I", CSRC,
           "--expt-relaxed-constexpr", "-o", tmp]
    if debug:
        cmd += ["-DSWA_DEBUG"]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv, debug="--debug" in sys.argv))
