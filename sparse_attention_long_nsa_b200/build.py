"""Build libnsa.so (sm_100a) in-tree with nvcc, and its checking variant.

    python -m sparse_attention_long_nsa_b200.build [--verbose-ptxas] [--force] [--no-check]

Each .cu under csrc/ is compiled to an object in _build/ (in parallel, only when
its sources changed) and linked into sparse_attention_long_nsa_b200/libnsa.so.
The checking variant libnsa_check.so is the same sources compiled with index
checks (-DNSA_DEBUG_BOUNDS), test fault injection (-DNSA_FAULT_INJECT, see
include/nsa_check.h) and a 20 ms limit on every bounded wait; only the tests load
it.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import hashlib
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libnsa.so")
CHECK_LIB = os.path.join(PKG, "libnsa_check.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I" + os.path.join(ROOT, "include")]
CHECK_DEFINES = ["-DNSA_DEBUG_BOUNDS", "-DNSA_FAULT_INJECT", "-DNSA_WAIT_LIMIT_NS=20000000ull"]


def _headers_digest() -> str:
    h = hashlib.sha1()
    for p in sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) +
                    glob.glob(os.path.join(ROOT, "include", "*.h"))):
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _compile(src: str, extra: list[str], hdr: str, force: bool, outdir: str) -> tuple[str, str]:
    obj = os.path.join(outdir, os.path.basename(src).replace(".cu", ".o"))
    stamp = obj + ".stamp"
    with open(src, "rb") as f:
        key = hashlib.sha1(f.read() + hdr.encode() + " ".join(FLAGS + extra).encode()).hexdigest()
    if not force and os.path.exists(obj) and os.path.exists(stamp) and open(stamp).read() == key:
        return obj, ""
    cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr}")
    with open(stamp, "w") as f:
        f.write(key)
    return obj, r.stderr


def _build_one(lib: str, outdir: str, extra: list[str], force: bool, quiet: bool, verbose: bool) -> str:
    os.makedirs(outdir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdr = _headers_digest()
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 4)) as ex:
        futs = [ex.submit(_compile, s, extra, hdr, force, outdir) for s in srcs]
        results = [f.result() for f in futs]
    if verbose or not quiet:
        for _, err in results:
            if err:
                sys.stderr.write(err)
    objs = [o for o, _ in results]
    newest = max(os.path.getmtime(o) for o in objs)
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < newest:
        cmd = [NVCC, *ARCH, "-shared", "-o", lib, *objs, "-lcudart"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stderr}")
    return lib


def build(verbose_ptxas: bool = False, force: bool = False, quiet: bool = True, check: bool = True) -> str:
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    _build_one(LIB, BUILD, extra, force or verbose_ptxas, quiet, verbose_ptxas)
    if check:
        build_check(force=force, quiet=quiet)
    return LIB


def build_check(force: bool = False, quiet: bool = True) -> str:
    """The checking variant (index checks, test fault injection, short wait limit)."""
    return _build_one(CHECK_LIB, os.path.join(BUILD, "check"), CHECK_DEFINES, force, quiet, False)


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--no-check", action="store_true", help="skip the checking variant")
    args = ap.parse_args()
    print(build(verbose_ptxas=args.verbose_ptxas, force=args.force, quiet=False, check=not args.no_check))
