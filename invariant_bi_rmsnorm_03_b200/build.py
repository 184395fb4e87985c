"""Builds the CUDA libraries in-tree for sm_100a.

    python -m invariant_bi_rmsnorm_03_b200.build            # both libraries
    python -m invariant_bi_rmsnorm_03_b200.build --force

Produces ``lib/libbi.so`` (batch-invariant build) and
``lib/libbi_variant.so`` (the variant-off build, ``-DBI_INVARIANT=0``, which
exists to measure what invariance costs).  Each translation unit is compiled
by nvcc with ``-gencode arch=compute_100a,code=sm_100a``; object files go to
``_build/`` and are rebuilt when a source or header is newer.
"""
from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBDIR = os.path.join(PKG, "lib")
BUILD = os.path.join(ROOT, "_build")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]

VARIANTS = {"libbi.so": 1, "libbi_variant.so": 0}


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) +
                  glob.glob(os.path.join(INCLUDE, "*.h")))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _run(cmd):
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("command failed: %s\n%s%s" % (" ".join(cmd), r.stdout, r.stderr))
    return r.stdout + r.stderr


def build(force: bool = False, verbose: bool = False, jobs: int | None = None) -> dict:
    """Compile both libraries; returns {library name: path}."""
    os.makedirs(LIBDIR, exist_ok=True)
    os.makedirs(BUILD, exist_ok=True)
    headers = _headers()
    jobs = jobs or min(16, (os.cpu_count() or 4))
    tasks, links = [], {}
    for lib, inv in VARIANTS.items():
        objs = []
        for src in _sources():
            obj = os.path.join(BUILD, "%s.inv%d.o" % (os.path.basename(src)[:-3], inv))
            objs.append(obj)
            if force or _stale(obj, [src] + headers):
                cmd = [NVCC] + ARCH + FLAGS + ["-DBI_INVARIANT=%d" % inv, "-c", src, "-o", obj]
                if verbose:
                    cmd.insert(1, "-Xptxas=-v")
                tasks.append(cmd)
        links[lib] = objs
    if tasks:
        with ThreadPoolExecutor(jobs) as ex:
            for out in ex.map(_run, tasks):
                if verbose and out.strip():
                    print(out)
    paths = {}
    for lib, objs in links.items():
        path = os.path.join(LIBDIR, lib)
        if force or _stale(path, objs):
            tmp = path + ".tmp%d" % os.getpid()
            _run([NVCC] + ARCH + ["-shared", "-o", tmp] + objs)
            os.replace(tmp, path)
        paths[lib] = path
    return paths


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true", help="print ptxas resource usage")
    a = ap.parse_args(argv)
    for k, v in build(force=a.force, verbose=a.verbose).items():
        print(k, "->", v)


if __name__ == "__main__":
    sys.exit(main())
