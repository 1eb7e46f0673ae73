"""Builds liblsa.so in-tree for sm_100a with nvcc (no GPU needed).

    python -m sparse_attention_decode_scan_b200.build [--force]

Objects go to _build/ at the repository root; the shared libraries are written
next to this file so the binding finds them:
  liblsa.so       the product library (include/lsa.h)
  liblsa_test.so  the same objects with abi.cu compiled with LSA_TEST_HOOKS,
                  which adds lsa_test_set_hooks (include/lsa_test.h); only the
                  tests load it
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJDIR = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "liblsa.so")
TEST_LIB = os.path.join(PKG, "liblsa_test.so")
HOOKED = "abi.cu"  # the one source whose test build differs

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I" + INCLUDE, "-I" + CSRC]


def nvcc() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found")
    return p


def _deps_mtime() -> float:
    files = glob.glob(os.path.join(CSRC, "*")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return max(os.path.getmtime(f) for f in files)


def build(force: bool = False, verbose: bool = False) -> str:
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    newest = _deps_mtime()
    if (not force and all(os.path.exists(p) and os.path.getmtime(p) >= newest for p in (LIB, TEST_LIB))):
        return LIB
    os.makedirs(OBJDIR, exist_ok=True)
    nv = nvcc()

    def compile_one(job):
        src, obj, extra = job
        cmd = [nv, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout, r.stderr, file=sys.stderr)
        return obj

    jobs = [(src, os.path.join(OBJDIR, os.path.basename(src) + ".o"), []) for src in sources]
    hooked = os.path.join(CSRC, HOOKED)
    jobs.append((hooked, os.path.join(OBJDIR, "abi_test_hooks.cu.o"), ["-DLSA_TEST_HOOKS"]))
    with ThreadPoolExecutor(max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
        objs = list(ex.map(compile_one, jobs))
    prod = objs[:-1]
    test = [o if os.path.basename(o) != HOOKED + ".o" else objs[-1] for o in prod]
    for out, ob in ((LIB, prod), (TEST_LIB, test)):
        tmp = out + ".tmp"
        r = subprocess.run([nv, *ARCH, "-shared", "-o", tmp, *ob], capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, out)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
