"""Build libloopvq.so in-tree for sm_100a with nvcc.

``python sub_bit_vq_b200/build.py`` compiles every source under ``csrc/``
into ``_build/`` and links ``sub_bit_vq_b200/libloopvq.so``. Objects are
rebuilt when their source, a header, or the flags changed.
"""

from __future__ import annotations

import concurrent.futures as cf
import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libloopvq.so")

# Test builds of the same sources: name -> extra nvcc flags. The range-check
# build checks the decode kernel's indices against their buffers; the
# short-wait build gives the tensor-core encoder no tries at all, so a test can
# watch the encoder report a timeout (it then waits, bounded, for the
# tensor cores before freeing their memory).
VARIANTS = {
    "rangecheck": ["-DLOOPVQ_RANGE_CHECK"],
    "shortwait": ["-DLOOPVQ_TC_SPIN=0"],
}


def variant_path(name: str) -> str:
    return os.path.join(PKG, f"libloopvq_{name}.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
              "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC] + ARCH


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libloopvq")
    return cand


def _headers_digest() -> str:
    h = hashlib.sha256()
    for d in (CSRC, INCLUDE):
        for f in sorted(os.listdir(d)):
            if f.endswith((".h", ".cuh")):
                with open(os.path.join(d, f), "rb") as fh:
                    h.update(f.encode() + fh.read())
    h.update(" ".join(NVCC_FLAGS).encode())
    return h.hexdigest()[:16]


def _sources() -> list[str]:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                  if f.endswith((".cu", ".cpp")))


def _compile(src: str, obj: str, extra: list[str]) -> None:
    cmd = [_nvcc(), "-c", src, "-o", obj] + NVCC_FLAGS + extra
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stdout}\n{r.stderr}")


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          variant: str | None = None) -> str:
    """Compile and link; returns the path of libloopvq.so (or of the test
    build `variant`, see VARIANTS)."""
    extra = list(extra or []) + (VARIANTS[variant] if variant else [])
    lib = variant_path(variant) if variant else LIB
    os.makedirs(BUILD, exist_ok=True)
    tag = _headers_digest() + hashlib.sha256(" ".join(extra).encode()).hexdigest()[:8]
    jobs = []
    objs = []
    for src in _sources():
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:12]
        obj = os.path.join(BUILD, f"{os.path.basename(src)}.{h}.{tag}.o")
        objs.append(obj)
        if force or not os.path.exists(obj):
            jobs.append((src, obj))
    if jobs:
        with cf.ThreadPoolExecutor(max_workers=min(8, len(jobs))) as ex:
            futs = [ex.submit(_compile, s, o, extra) for s, o in jobs]
            for f in futs:
                f.result()
    stamp = os.path.join(BUILD, f"link{'.' + variant if variant else ''}.stamp")
    want = "\n".join(objs)
    have = open(stamp).read() if os.path.exists(stamp) else ""
    if force or jobs or want != have or not os.path.exists(lib):
        tmp = lib + ".tmp"
        cmd = [_nvcc(), "-shared", "-o", tmp] + objs + ARCH + ["-lcudart"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib)
        with open(stamp, "w") as fh:
            fh.write(want)
    if verbose:
        print(f"built {lib} ({len(jobs)} objects recompiled)")
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    for name in VARIANTS:
        build(force="--force" in sys.argv, verbose=True, variant=name)
