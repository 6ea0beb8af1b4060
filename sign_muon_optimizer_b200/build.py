"""Build libsignmuon.so in-tree with nvcc for sm_100a.

    python sign_muon_optimizer_b200/build.py [--force]

Every CUDA source is compiled with ``-gencode arch=compute_100a,code=sm_100a
-lineinfo -O3`` and linked with the static CUDA runtime; the library has no
PyTorch dependency.  Objects go to ``_build/`` beside the package.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libsignmuon.so")

SOURCES = ["kernels_elem.cu", "kernels_ternary.cu", "ns_simt.cu", "ns_tc.cu", "signmuon_api.cu", "noalloc.cu",
           "plan.cpp"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-I" + INCLUDE,
                     "--expt-relaxed-constexpr"]
EXTRA = [f for f in os.environ.get("SIGNMUON_NVCC_DEFINES", "").split() if f.startswith("-D")]


def _nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _headers():
    out = [os.path.join(INCLUDE, "signmuon.h")]
    out += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    return out


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, out: str = LIB, build_dir: str = BUILD) -> str:
    """Compile (only stale objects unless force) into ``build_dir`` and link
    ``out``.  SIGNMUON_NVCC_DEFINES may add -D options (tuning experiments,
    which should use their own build_dir and out)."""
    os.makedirs(build_dir, exist_ok=True)
    nvcc = _nvcc()
    hdrs = _headers()
    objs, jobs = [], []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(build_dir, src + ".o")
        objs.append(o)
        if force or _stale(o, [s] + hdrs):
            cmd = [nvcc] + NVCC_FLAGS + EXTRA + ["-x", "cu" if src.endswith(".cu") else "c++", "-c", s, "-o", o]
            if src.endswith(".cpp"):
                cmd = [nvcc] + ["-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-I" + INCLUDE] + EXTRA + ["-c", s, "-o", o]
            jobs.append(cmd)
    with cf.ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
        for cmd, res in zip(jobs, ex.map(lambda c: subprocess.run(c, capture_output=True, text=True), jobs)):
            if verbose or res.returncode:
                sys.stderr.write(" ".join(cmd) + "\n" + res.stdout + res.stderr)
            if res.returncode:
                raise RuntimeError("nvcc failed for " + cmd[-3])
    if force or jobs or _stale(out, objs):
        cmd = [nvcc] + ARCH + ["-shared", "-cudart", "static", "-o", out] + objs
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode:
            sys.stderr.write(" ".join(cmd) + "\n" + res.stdout + res.stderr)
            raise RuntimeError("link of libsignmuon.so failed")
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
