"""Build libfbk.so (the C-ABI CUDA library) in-tree for sm_100a.

    python -m cached_block_attention_b200.build [--verbose]

Compiles every csrc/*.cu with nvcc for sm_100a only and links them into
cached_block_attention_b200/libfbk.so (CUDA runtime linked statically, no
libcuda link: the tensor-map encoder is fetched through the runtime's driver
entry-point query). Objects go to _build/ at the repository root.

It also links libfbk_testhooks.so, the test build: the same objects except
the prefix kernel's and the FP8 quantisation's, which are compiled with
FBK_TEST_HOOKS so that a test can shorten the prefix kernel's bounded waits
and withhold one of its loads, and run the FP8 kernel's per-group scale step
on given values (include/fbk_test_hooks.h). Only the bounded-wait and the
FP8 scale tests load it.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libfbk.so")
TEST_LIB = os.path.join(PKG, "libfbk_testhooks.so")
HOOKED = ("prefix_tc.cu", "fp8_quant.cu")  # the sources the test build compiles differently

SOURCES = ["abi.cu", "prefix_tc.cu", "prefix_fp32.cu", "split_reduce.cu", "block_merge.cu",
           "commit.cu", "full_ref.cu", "fp8_quant.cu", "facache_rows.cu", "sparse_prefix.cu"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
                "--expt-relaxed-constexpr", "-I", INCLUDE]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _newer(target: str, deps) -> bool:
    if not os.path.exists(target):
        return False
    t = os.path.getmtime(target)
    return all(os.path.getmtime(d) <= t for d in deps)


def build(verbose: bool = False, force: bool = False, ptxas_info: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    headers += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    cc = nvcc()

    def compile_one(job):
        src, hooks = job
        path = os.path.join(CSRC, src)
        obj = os.path.join(BUILD, src.replace(".cu", "_hooks.o" if hooks else ".o"))
        if not force and not ptxas_info and _newer(obj, [path] + headers):
            return obj, ""
        cmd = ([cc] + FLAGS + (["-DFBK_TEST_HOOKS"] if hooks else []) + (["-Xptxas", "-v"] if ptxas_info else [])
               + ["-c", path, "-o", obj])
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        return obj, r.stderr

    jobs = [(src, False) for src in SOURCES] + [(src, True) for src in HOOKED]
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(compile_one, jobs))
    objs = {job: o for job, (o, _) in zip(jobs, results)}
    if verbose or ptxas_info:
        for (src, hooks), (_, log) in zip(jobs, results):
            if log.strip() and not hooks:
                print(f"--- {src}\n{log}")

    def link(target, parts):
        if force or not _newer(target, parts):
            cmd = [cc] + ARCH + ["-shared", "-o", target] + parts
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")

    link(LIB, [objs[(s, False)] for s in SOURCES])
    link(TEST_LIB, [objs[(s, s in HOOKED)] for s in SOURCES])
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers/spills per kernel")
    a = ap.parse_args()
    print(build(verbose=a.verbose, force=a.force, ptxas_info=a.ptxas_info))
