"""Build libssm_causal.so in-tree with nvcc for sm_100a.

    python -m state_space_model_causal_b200.build [--force] [--verbose]

Each translation unit under ``csrc/`` is compiled to an object in
``_build/`` (git-ignored) and linked into
``state_space_model_causal_b200/libssm_causal.so``.  Objects are rebuilt when
their source or any header is newer.  ``-Xptxas -v`` output (registers,
spills, shared memory per kernel) is written to ``_build/ptxas.txt``.

A second library, ``libssm_causal_testhooks.so``, is linked from the same
objects except that the translation units with failure-test switches
(``TEST_HOOK_SOURCES``) are compiled again with ``-DSSM_TEST_HOOKS``; only the
GPU failure tests load it.  The product library has no such switches.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libssm_causal.so")
TEST_LIB = os.path.join(PKG, "libssm_causal_testhooks.so")
TEST_HOOK_SOURCES = ("ssu.cu", "scan_bal.cu", "api.cpp")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I", INCLUDE,
                     "-Xptxas", "-v"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _headers():
    return glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _compile(src: str, force: bool, test_hooks: bool = False):
    obj = os.path.join(BUILD, os.path.basename(src) + (".testhooks.o" if test_hooks else ".o"))
    newest = max([os.path.getmtime(src)] + [os.path.getmtime(h) for h in _headers()])
    if not force and os.path.exists(obj) and os.path.getmtime(obj) >= newest:
        return obj, ""
    extra = ["-DSSM_TEST_HOOKS"] if test_hooks else []
    cmd = [_nvcc()] + NVCC_FLAGS + extra + ["-c", src, "-o", obj]
    if src.endswith(".cpp"):
        cmd = [_nvcc()] + ARCH + ["-O3", "-std=c++17", "-Xcompiler", "-fPIC,-Wall", "-I", INCLUDE] + extra + \
            ["-x", "c++", "-c", src, "-o", obj]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{res.stdout}\n{res.stderr}")
    return obj, res.stderr


def _link(lib: str, objs, force: bool):
    newest_obj = max(os.path.getmtime(o) for o in objs)
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < newest_obj:
        tmp = lib + f".tmp{os.getpid()}"
        cmd = [_nvcc()] + ARCH + ["-shared", "-o", tmp] + list(objs) + ["-lcudart_static"]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"link failed:\n{res.stdout}\n{res.stderr}")
        os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every CUDA/C++ source, link libssm_causal.so and the failure-test
    build libssm_causal_testhooks.so; return the product library's path."""
    os.makedirs(BUILD, exist_ok=True)
    srcs = _sources()
    jobs = [(s, False) for s in srcs] + [(s, True) for s in srcs if os.path.basename(s) in TEST_HOOK_SOURCES]
    with cf.ThreadPoolExecutor(max_workers=min(8, len(jobs))) as ex:
        results = list(ex.map(lambda j: _compile(j[0], force, j[1]), jobs))
    objs = {j: o for j, (o, _) in zip(jobs, results)}
    logs = "".join(l for (_, hooks), (_, l) in zip(jobs, results) if l and not hooks)
    if logs:
        with open(os.path.join(BUILD, "ptxas.txt"), "w") as f:
            f.write(logs)
        if verbose:
            sys.stderr.write(logs)
    _link(LIB, [objs[(s, False)] for s in srcs], force)
    _link(TEST_LIB, [objs[(s, os.path.basename(s) in TEST_HOOK_SOURCES)] for s in srcs], force)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
