"""Build libpagedkv.so in-tree with nvcc for sm_100a.

Usage: python -m paged_kv_cache_336_b200.build [--force] [--verbose-ptxas] [--nvtx]

Objects go to <repo>/_build/ (<repo>/_build/nvtx/ for the NVTX variant), the
shared library next to this file. A source is recompiled when it or any
header in csrc/ or include/ is newer than its object. nvcc cross-compiles; no
GPU is needed.

--nvtx (or PAGEDKV_NVTX=1 in the environment) compiles NVTX ranges around
every C-ABI call that enqueues GPU work (PAGEDKV_NVTX defined); the default
build has none.
"""

from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libpagedkv.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O3",
          f"-I{INCLUDE}", f"-I{CSRC}"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                  if f.endswith((".cu", ".cpp")))


def headers_mtime() -> float:
    t = 0.0
    for d in (CSRC, INCLUDE):
        for f in os.listdir(d):
            if f.endswith((".h", ".cuh", ".hpp")):
                t = max(t, os.path.getmtime(os.path.join(d, f)))
    return t


def _compile(src: str, obj: str, ptxas_verbose: bool, defines=()) -> tuple[str, str]:
    cmd = [nvcc(), *ARCH, *COMMON, *(f"-D{d}" for d in defines), "-c", src, "-o", obj]
    if ptxas_verbose and src.endswith(".cu"):
        cmd += ["-Xptxas", "-v"]
    p = subprocess.run(cmd, capture_output=True, text=True)
    if p.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{' '.join(cmd)}\n{p.stdout}\n{p.stderr}")
    return src, p.stdout + p.stderr


def build(force: bool = False, ptxas_verbose: bool = False, jobs: int | None = None,
          nvtx: bool | None = None) -> str:
    if nvtx is None:
        nvtx = os.environ.get("PAGEDKV_NVTX") == "1"
    build_dir = os.path.join(BUILD, "nvtx") if nvtx else BUILD
    defines = ("PAGEDKV_NVTX=1",) if nvtx else ()
    os.makedirs(build_dir, exist_ok=True)
    hdr = headers_mtime()
    todo, objs = [], []
    for src in sources():
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        objs.append(obj)
        if force or not os.path.exists(obj) or os.path.getmtime(obj) < max(os.path.getmtime(src), hdr):
            todo.append((src, obj))
    logs = []
    if todo:
        with cf.ThreadPoolExecutor(max_workers=jobs or min(len(todo), os.cpu_count() or 4)) as ex:
            for src, log in ex.map(lambda so: _compile(so[0], so[1], ptxas_verbose, defines), todo):
                if log.strip():
                    logs.append(f"== {os.path.basename(src)}\n{log}")
    # which variant the library was last linked from
    stamp = os.path.join(BUILD, "variant")
    variant = "nvtx" if nvtx else "plain"
    try:
        with open(stamp) as f:
            linked = f.read().strip()
    except OSError:
        linked = ""
    relink = bool(todo) or not os.path.exists(LIB) or linked != variant or any(
        os.path.getmtime(o) > os.path.getmtime(LIB) for o in objs)
    if relink:
        tmp = LIB + ".tmp"
        cmd = [nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", tmp, *objs]
        p = subprocess.run(cmd, capture_output=True, text=True)
        if p.returncode != 0:
            raise RuntimeError(f"link failed:\n{' '.join(cmd)}\n{p.stdout}\n{p.stderr}")
        os.replace(tmp, LIB)
        with open(stamp, "w") as f:
            f.write(variant)
    if ptxas_verbose and logs:
        with open(os.path.join(build_dir, "ptxas.log"), "w") as f:
            f.write("\n".join(logs))
    return LIB


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--nvtx", action="store_true", help="compile NVTX ranges around the C-ABI calls")
    args = ap.parse_args(argv)
    lib = build(force=args.force, ptxas_verbose=args.verbose_ptxas, nvtx=args.nvtx or None)
    print(lib)
    return 0


if __name__ == "__main__":
    sys.exit(main())
