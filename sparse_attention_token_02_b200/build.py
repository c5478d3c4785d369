"""Builds the CUDA library of the indexer for sm_100a (nvcc; no GPU needed).

    python -m sparse_attention_token_02_b200.build [--jobs N] [--verbose]

Compiles every ``csrc/*.cu`` to an object with
``-gencode arch=compute_100a,code=sm_100a -lineinfo -O3`` and links them into
``libdsa_indexer.so`` next to this file (static CUDA runtime, so loading the
library needs only the driver; only the ``dsa_*`` C symbols are exported).
Objects are rebuilt when a source or header is newer.
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
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libdsa_indexer.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
          "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _headers() -> list[str]:
    return glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(jobs: int = 8, verbose: bool = False, extra: list[str] | None = None, out_dir: str | None = None) -> str:
    """Build the library; `extra` nvcc flags and `out_dir` (objects and .so) serve tuning builds."""
    build_dir = os.path.join(out_dir, "_build") if out_dir else BUILD
    lib_path = os.path.join(out_dir, "libdsa_indexer.so") if out_dir else LIB
    os.makedirs(build_dir, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = _headers()
    cmds = []
    objs = []
    for src in sources:
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if _stale(obj, [src] + headers):
            cmds.append([nvcc(), *ARCH, *CFLAGS, *(extra or []), "-c", src, "-o", obj])

    def run(cmd):
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout, r.stderr, flush=True)

    with cf.ThreadPoolExecutor(max_workers=max(1, jobs)) as ex:
        list(ex.map(run, cmds))
    if cmds or _stale(lib_path, objs):
        run([nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", lib_path, *objs])
    return lib_path


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--jobs", type=int, default=8)
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers / shared memory per kernel")
    a = ap.parse_args(argv)
    extra = ["-Xptxas", "-v"] if a.ptxas_info else None
    if extra:
        for f in glob.glob(os.path.join(BUILD, "*.o")):
            os.remove(f)
    print(build(a.jobs, a.verbose or a.ptxas_info, extra))
    return 0


if __name__ == "__main__":
    sys.exit(main())
