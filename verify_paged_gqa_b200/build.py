"""Builds libtfpaged.so (the C-ABI CUDA library) in place, for sm_100a only.

    python -m verify_paged_gqa_b200.build [--verbose]

nvcc compiles each translation unit under csrc/ to an object in _build/ and
links them into verify_paged_gqa_b200/libtfpaged.so.  ``--verbose`` adds
``-Xptxas -v`` (registers, spills, shared memory per kernel) to the log.
"""
from __future__ import annotations

import concurrent.futures
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build", "tfpaged")
LIB = os.path.join(HERE, "libtfpaged.so")
SOURCES = ["tf_paged.cu", "kv_put.cu", "kv_copy.cu", "attn_simt.cu", "attn_prompt.cu", "attn_pm.cu",
           "attn_merge.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "--expt-relaxed-constexpr",
         "-Xcompiler", "-fPIC,-fvisibility=hidden", "-I", os.path.join(ROOT, "include")]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; the CUDA library cannot be built")
    return cand


def _deps():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(ROOT, "include", "tf_paged.h"))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _deps())


# host-compiler flags of the sanitizer build (one per -Xcompiler: nvcc splits
# an -Xcompiler value at commas)
SANITIZE = ["-fsanitize=address", "-fsanitize=undefined", "-fno-sanitize-recover=undefined",
            "-fno-omit-frame-pointer"]


def build(verbose: bool = False, force: bool = False, sanitize: bool = False) -> str:
    """Compile and link the library; returns its path.  ``sanitize`` builds a
    separate copy (_build/asan/libtfpaged_asan.so) whose host code carries
    AddressSanitizer and UndefinedBehaviorSanitizer (device code is
    unchanged; the process that loads it must preload libasan)."""
    if not sanitize and not force and not verbose and up_to_date():
        return LIB
    build_dir = os.path.join(ROOT, "_build", "asan") if sanitize else BUILD
    lib = os.path.join(build_dir, "libtfpaged_asan.so") if sanitize else LIB
    os.makedirs(build_dir, exist_ok=True)
    cc = nvcc()
    extra = ["-Xptxas", "-v"] if verbose else []
    if sanitize:
        extra += [f"-Xcompiler={f}" for f in SANITIZE] + ["-g"]

    def compile_one(src):
        obj = os.path.join(build_dir, src.replace(".cu", ".o"))
        cmd = [cc, *ARCH, *FLAGS, *extra, "-c", os.path.join(CSRC, src), "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        return obj, r.stdout + r.stderr

    with concurrent.futures.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        results = list(ex.map(compile_one, SOURCES))
    log = "".join(out for _, out in results)
    with open(os.path.join(build_dir, "ptxas.log"), "w") as f:
        f.write(log)
    tmp = lib + f".tmp{os.getpid()}"
    link_extra = ["-Xcompiler=-fsanitize=address", "-Xcompiler=-fsanitize=undefined"] if sanitize else []
    cmd = [cc, *ARCH, "-shared", *link_extra, "-o", tmp, *[o for o, _ in results], "-lcudart"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    if verbose:
        sys.stdout.write(log)
    return lib


if __name__ == "__main__":
    build(verbose="--verbose" in sys.argv, force=True)
