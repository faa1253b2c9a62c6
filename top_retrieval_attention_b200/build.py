"""Build the in-tree shared libraries with nvcc for sm_100a.

  libra.so        top_retrieval_attention_b200/csrc/*.cu   (the product: kernels + C ABI)
  libra_synth.so  synth/csrc/synth.cu                      (device fill of synthetic inputs)

Usage: python -m top_retrieval_attention_b200.build [--force] [--verbose]
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
BUILD = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O3",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]

TARGETS = {
    "libra": (sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu"))),
              os.path.join(PKG, "libra.so"),
              sorted(glob.glob(os.path.join(PKG, "csrc", "*.cuh")) +
                     glob.glob(os.path.join(PKG, "csrc", "*.h")) +
                     [os.path.join(ROOT, "include", "ra.h")])),
    "libra_synth": ([os.path.join(ROOT, "synth", "csrc", "synth.cu")],
                    os.path.join(ROOT, "synth", "libra_synth.so"),
                    [os.path.join(ROOT, "include", "ra_synth.h")]),
}


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _stale(out: str, deps: list[str]) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def _run(cmd: list[str], verbose: bool) -> str:
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"command failed ({r.returncode}): {' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    return r.stdout + r.stderr


def build_target(name: str, force: bool = False, verbose: bool = False, ptxas_v: bool = False) -> str:
    srcs, out, hdrs = TARGETS[name]
    if not force and not _stale(out, srcs + hdrs + [os.path.abspath(__file__)]):
        return out
    os.makedirs(BUILD, exist_ok=True)
    nv = nvcc()
    extra = ["-Xptxas", "-v"] if ptxas_v else []

    def compile_one(src: str) -> tuple[str, str]:
        obj = os.path.join(BUILD, f"{name}_{os.path.splitext(os.path.basename(src))[0]}.o")
        log = _run([nv, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj], verbose)
        return obj, log

    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        results = list(ex.map(compile_one, srcs))
    if ptxas_v:
        for _, log in results:
            sys.stdout.write(log)
    objs = [o for o, _ in results]
    tmp = out + ".tmp"
    _run([nv, *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"], verbose)
    os.replace(tmp, out)
    return out


def build_all(force: bool = False, verbose: bool = False, ptxas_v: bool = False) -> list[str]:
    return [build_target(n, force, verbose, ptxas_v) for n in TARGETS]


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true", help="print register / smem usage")
    a = ap.parse_args()
    for p in build_all(a.force or a.ptxas_v, a.verbose, a.ptxas_v):
        print(p)


if __name__ == "__main__":
    main()
