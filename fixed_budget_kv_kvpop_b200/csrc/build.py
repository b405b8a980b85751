"""Builds libkvpop.so (all CUDA sources of the package) in-tree for sm_100a.

Usage: python fixed_budget_kv_kvpop_b200/csrc/build.py [--force] [-v]
(run by file path: importing the package would load the library being rebuilt)
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(HERE)
ROOT = os.path.dirname(PKG)
SOURCES = ["kvpop_api.cu", "kvpop_decode.cu", "kvpop_prefill.cu", "kvpop_prefill_attn.cu"]
HEADERS = ["kvpop_internal.cuh", "kvpop_prefill_attn.cuh", os.path.join(ROOT, "include", "kvpop.h")]
OUT = os.path.join(PKG, "libkvpop.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-shared", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
         "-I" + os.path.join(ROOT, "include")]


def _stale() -> bool:
    if not os.path.exists(OUT):
        return True
    t = os.path.getmtime(OUT)
    deps = [os.path.join(HERE, s) for s in SOURCES] + [os.path.join(HERE, h) if not os.path.isabs(h) else h
                                                      for h in HEADERS] + [__file__]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, out: str = OUT, defines=()) -> str:
    if out == OUT and not defines and not force and not _stale():
        return OUT
    cmd = [NVCC] + FLAGS + ["-D" + d for d in defines] + [os.path.join(HERE, s) for s in SOURCES] + ["-o", out + ".tmp"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libkvpop.so")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
