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
SOURCES = ["kvpop_api.cu", "kvpop_decode.cu", "kvpop_prefill.cu", "kvpop_prefill_attn.cu", "kvpop_mlstm.cu"]
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
    """Compiles every source to an object in parallel, then links the shared
    library (each translation unit's device code is self-contained, so no
    device link step is needed)."""
    if out == OUT and not defines and not force and not _stale():
        return OUT
    import tempfile
    from concurrent.futures import ThreadPoolExecutor
    tmp = tempfile.mkdtemp(prefix="kvpop_build_")
    extra = ["-D" + d for d in defines] + (["-Xptxas=-v"] if verbose else [])
    compile_flags = [f for f in FLAGS if f != "-shared"]

    def compile_one(src):
        obj = os.path.join(tmp, os.path.splitext(src)[0] + ".o")
        cmd = [NVCC] + compile_flags + extra + ["-c", os.path.join(HERE, src), "-o", obj]
        return obj, subprocess.run(cmd, capture_output=True, text=True)

    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        results = list(ex.map(compile_one, SOURCES))
    for obj, res in results:
        if res.returncode != 0:
            sys.stderr.write(res.stdout + res.stderr)
            raise RuntimeError("nvcc failed building libkvpop.so")
        if verbose:
            sys.stderr.write(res.stderr)
    link = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-Xcompiler", "-fPIC"] + \
        [obj for obj, _ in results] + ["-o", out + ".tmp"]
    res = subprocess.run(link, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed linking libkvpop.so")
    os.replace(out + ".tmp", out)
    for obj, _ in results:
        os.remove(obj)
    os.rmdir(tmp)
    return out


TEST_HOOKS_OUT = os.path.join(PKG, "libkvpop_testhooks.so")
# The failure-injection build: kvpop_debug_set_hook works, and the decode
# kernel's merge-queue waits give up after 50 ms instead of 2 s.
TEST_HOOKS_DEFINES = ("KVPOP_TEST_HOOKS", "KVPOP_MERGE_WAIT_LIMIT_NS=50000000ull")


def build_test_hooks(force: bool = False) -> str:
    if not force and os.path.exists(TEST_HOOKS_OUT):
        t = os.path.getmtime(TEST_HOOKS_OUT)
        deps = [os.path.join(HERE, s) for s in SOURCES] + [os.path.join(HERE, h) if not os.path.isabs(h) else h
                                                          for h in HEADERS] + [__file__]
        if all(os.path.getmtime(p) <= t for p in deps):
            return TEST_HOOKS_OUT
    return build(out=TEST_HOOKS_OUT, defines=TEST_HOOKS_DEFINES)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
    if "--test-hooks" in sys.argv:
        print(build_test_hooks(force="--force" in sys.argv))
