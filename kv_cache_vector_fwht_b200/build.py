"""Build libtq.so in-tree for sm_100a with nvcc (python kv_cache_vector_fwht_b200/build.py).

Objects go to _build/ at the repository root; the shared library lands next to this file so
that it travels with the source tree. Rebuilds only sources newer than their objects.
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libtq.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

SOURCES = ["tq_api.cu", "quantize.cu", "keys_tc.cu", "dequant.cu", "decode.cu", "decode_prod.cu",
           "decode_mse.cu", "decode_grp.cu", "append.cu",
           "tq_host.cpp"]
HEADERS = ["tq_internal.h", "tq_device.cuh", "decode_kernel.cuh", os.path.join("..", "..", "include", "tq.h")]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O3",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def _newest_header() -> float:
    return max(os.path.getmtime(os.path.join(CSRC, h)) for h in HEADERS)


def _compile(src: str, verbose: bool) -> str:
    out = os.path.join(OBJ, os.path.splitext(src)[0] + ".o")
    path = os.path.join(CSRC, src)
    if (os.path.exists(out) and os.path.getmtime(out) > os.path.getmtime(path)
            and os.path.getmtime(out) > _newest_header()):
        return out
    cmd = [NVCC, *ARCH, *FLAGS, "-c", path, "-o", out]
    if src.endswith(".cpp"):
        cmd = ["g++", "-O3", "-std=c++17", "-fPIC", "-I", "/usr/local/cuda/include",
               "-I", os.path.join(ROOT, "include"), "-c", path, "-o", out]
    if verbose and src.endswith(".cu"):
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose:
        sys.stderr.write(r.stderr)
    return out


def build(verbose: bool = False) -> str:
    os.makedirs(OBJ, exist_ok=True)
    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose), SOURCES))
    if not os.path.exists(LIB) or any(os.path.getmtime(o) > os.path.getmtime(LIB) for o in objs):
        cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", "-o", LIB, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
