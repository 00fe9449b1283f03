"""Build libsplitkv.so (sm_100a) in-tree with nvcc.

    python -m split_kv_lse_splitkv_b200.build [--verbose-ptxas]

Each .cu under csrc/ is compiled to an object in parallel, then linked into
split_kv_lse_splitkv_b200/libsplitkv.so with the CUDA runtime linked statically,
so the library has no dependency on a particular libcudart and loads on a
machine without a GPU (the driver is only needed when a call launches work).
"""
from __future__ import annotations

import concurrent.futures
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libsplitkv.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
SOURCES = ["abi.cu", "cost.cu", "plan.cu", "fwd_simt.cu", "fwd_tc.cu", "fwd_tc2.cu", "merge.cu", "bwd.cu", "bwd_tc.cu"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def source_digest() -> str:
    """sha256 (hex) of the library's sources: every .cu/.cuh/.h under csrc/ and include/splitkv.h, by
    relative name and content, in name order. Compiled into libsplitkv.so as its build id."""
    import hashlib
    h = hashlib.sha256()
    files = [("csrc/" + f, os.path.join(CSRC, f)) for f in sorted(os.listdir(CSRC)) if f.endswith((".cu", ".cuh", ".h"))]
    files.append(("include/splitkv.h", os.path.join(os.path.dirname(HERE), "include", "splitkv.h")))
    for rel, path in files:
        with open(path, "rb") as fh:
            h.update(rel.encode() + b"\0" + fh.read() + b"\0")
    return h.hexdigest()


def _newer(target: str, deps) -> bool:
    if not os.path.exists(target):
        return False
    t = os.path.getmtime(target)
    return all(os.path.getmtime(d) <= t for d in deps)


def build(verbose_ptxas: bool = False, force: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    headers.append(os.path.join(os.path.dirname(HERE), "include", "splitkv.h"))
    flags = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden",
                    "-I" + os.path.join(os.path.dirname(HERE), "include")]
    if verbose_ptxas:
        flags += ["-Xptxas", "-v"]
    nv = nvcc()
    # abi.cu carries the build id: it is recompiled whenever any source differs from the last build's.
    digest = source_digest()
    digest_file = os.path.join(BUILD, "source_digest.txt")
    last = open(digest_file).read().strip() if os.path.exists(digest_file) else ""

    def compile_one(src):
        path = os.path.join(CSRC, src)
        obj = os.path.join(BUILD, src.replace(".cu", ".o"))
        stale_id = src == "abi.cu" and last != digest
        if not force and not verbose_ptxas and not stale_id and _newer(obj, [path] + headers):
            return obj, ""
        extra = [f'-DSPLITKV_SOURCE_SHA="{digest}"'] if src == "abi.cu" else []
        cmd = [nv, *flags, *extra, "-c", path, "-o", obj]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{res.stdout}\n{res.stderr}")
        return obj, res.stderr

    with concurrent.futures.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        results = list(ex.map(compile_one, SOURCES))
    if verbose_ptxas:
        for (obj, log), src in zip(results, SOURCES):
            print(f"== {src}\n{log}")
    objs = [o for o, _ in results]
    if force or verbose_ptxas or not _newer(LIB, objs):
        cmd = [nv, *ARCH, "-shared", "-cudart", "static", "-o", LIB, *objs]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"link failed:\n{res.stdout}\n{res.stderr}")
    with open(digest_file, "w") as fh:
        fh.write(digest + "\n")
    return LIB


if __name__ == "__main__":
    print(build(verbose_ptxas="--verbose-ptxas" in sys.argv, force="--force" in sys.argv))
