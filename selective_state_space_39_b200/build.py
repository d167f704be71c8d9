"""Build libssmscan.so (the C-ABI library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
SOURCES = [os.path.join(CSRC, f) for f in ("ssm_scan_kernels.cu", "ssm_scan_bwd.cu",
                                           "ssm_conv1d.cu", "ssm_seqpar.cu", "ssm_ssd.cu",
                                           "ssm_ssd_tc.cu", "ssm_ssd_decode.cu",
                                           "ssm_api.cu")]
HEADERS = [os.path.join(CSRC, f) for f in ("ssm_device.cuh", "ssm_internal.h",
                                            "ssm_bwd_internal.h", "ssm_conv_internal.h",
                                            "ssm_seqpar_internal.h", "ssm_ssd_internal.h", "ssm_tc.cuh",
                                            "ssm_ssd_decode_internal.h")] + [
    os.path.join(os.path.dirname(HERE), "include", "ssm_scan.h")]
LIB_PATH = os.path.join(HERE, "libssmscan.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
         "--expt-relaxed-constexpr"]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libssmscan.so")
    return cand


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(s) <= t for s in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every source to an object in parallel, then link the shared
    library (same flags as one nvcc call over all sources)."""
    if not force and up_to_date():
        return LIB_PATH
    from concurrent.futures import ThreadPoolExecutor
    obj_dir = os.path.join(HERE, "_build")
    os.makedirs(obj_dir, exist_ok=True)
    compile_flags = [f for f in FLAGS if f != "-shared"]
    tag = "%d" % os.getpid()
    objs = [os.path.join(obj_dir, os.path.basename(src) + "." + tag + ".o") for src in SOURCES]

    def compile_one(pair):
        src, obj = pair
        cmd = [nvcc()] + ARCH + compile_flags + ["-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.run(cmd, check=True)

    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        list(ex.map(compile_one, zip(SOURCES, objs)))
    tmp = LIB_PATH + ".tmp." + tag
    cmd = [nvcc()] + ARCH + ["-shared", "-Xcompiler", "-fPIC", "-o", tmp] + objs
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB_PATH)
    for o in objs:
        os.remove(o)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
