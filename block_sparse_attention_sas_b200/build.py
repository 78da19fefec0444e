"""Build the SAS CUDA library (libsas_b200.so) in the package directory.

Each csrc/*.cu compiles to an object for sm_100a (nvcc -gencode
arch=compute_100a,code=sm_100a -lineinfo -O3), in parallel, and the objects
link into one shared library with the CUDA runtime linked statically. Nothing
links against libcuda: the driver entry points the library needs are fetched
at run time, so the library also loads on machines without a GPU driver.

Run as ``python -m block_sparse_attention_sas_b200.build`` or call build().
"""
from __future__ import annotations

import hashlib
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OUT = os.path.join(PKG, "libsas_b200.so")
BUILD_DIR = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVFLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O3", "--expt-relaxed-constexpr",
           "-Xptxas", "-warn-spills"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the SAS CUDA library cannot be built")


def _sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _headers():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    hs.append(os.path.join(ROOT, "include", "sas.h"))
    return sorted(hs)


def _digest(paths, extra=""):
    h = hashlib.sha256(extra.encode())
    for p in paths:
        h.update(p.encode())
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def build(verbose: bool = False, force: bool = False, jobs: int | None = None) -> str:
    """Compile every CUDA source for sm_100a and link libsas_b200.so; returns its path."""
    nvcc = _nvcc()
    os.makedirs(BUILD_DIR, exist_ok=True)
    hdr = _digest(_headers(), " ".join(ARCH + NVFLAGS))
    stamp = os.path.join(BUILD_DIR, "lib.stamp")
    srcs = _sources()
    full = _digest(srcs, hdr)
    if not force and os.path.exists(OUT) and os.path.exists(stamp):
        if open(stamp).read().strip() == full:
            return OUT

    def compile_one(src):
        obj = os.path.join(BUILD_DIR, os.path.basename(src)[:-3] + ".o")
        ostamp = obj + ".stamp"
        key = _digest([src], hdr)
        if not force and os.path.exists(obj) and os.path.exists(ostamp) and \
                open(ostamp).read().strip() == key:
            return obj, ""
        cmd = [nvcc, *ARCH, *NVFLAGS, "-I", os.path.join(ROOT, "include"), "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        with open(ostamp, "w") as f:
            f.write(key)
        return obj, r.stdout + r.stderr

    with ThreadPoolExecutor(jobs or min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(compile_one, srcs))
    for obj, log in results:
        if verbose and log.strip():
            print(log, file=sys.stderr)
    tmp = OUT + ".tmp"
    cmd = [nvcc, *ARCH, "-shared", "-o", tmp, *[o for o, _ in results], "-lpthread"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, OUT)
    with open(stamp, "w") as f:
        f.write(full)
    return OUT


if __name__ == "__main__":
    print(build(verbose=True, force="--force" in sys.argv))
