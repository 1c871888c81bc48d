"""Build of the in-tree CSA2 library (``lib/libcsa2.so``) for sm_100a with nvcc."""
from __future__ import annotations

import glob
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "lib", "libcsa2.so")
# The same library with test hooks (short wait limits, a stall that makes a
# bounded wait run out): loaded only by tests/test_gpu_timeout.py.
TEST_LIB = os.path.join(PKG, "lib", "libcsa2_test.so")
TEST_HOOK_SOURCES = ("attention.cu", "score_mma.cu")
# Access-pattern ceilings (kernels that only move bytes in the CSA2 kernels'
# patterns): a measurement aid loaded by the benchmark, not part of libcsa2.so.
CEIL_SRC = os.path.join(PKG, "ceilings", "ceilings.cu")
CEIL_LIB = os.path.join(PKG, "lib", "libcsa2_ceilings.so")

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC",
    "-Xptxas", "-v",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs() -> list[str]:
    return (sources() + glob.glob(os.path.join(CSRC, "*.cuh")) +
            glob.glob(os.path.join(ROOT, "include", "*.h")) + [os.path.abspath(__file__)])


def up_to_date() -> bool:
    if not all(os.path.exists(p) for p in (LIB, TEST_LIB, CEIL_LIB)):
        return False
    t = min(os.path.getmtime(LIB), os.path.getmtime(TEST_LIB), os.path.getmtime(CEIL_LIB))
    return all(os.path.getmtime(p) <= t for p in _inputs() + [CEIL_SRC])


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every csrc/*.cu for sm_100a and link libcsa2.so (in-tree)."""
    if not force and up_to_date():
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    os.makedirs(os.path.dirname(LIB), exist_ok=True)

    def compile_one(job: tuple[str, bool]) -> tuple[str, str]:
        src, hooks = job
        obj = os.path.join(BUILD, os.path.basename(src) + (".test.o" if hooks else ".o"))
        cmd = ["nvcc", *NVCC_FLAGS, *(["-DCSA2_TEST_HOOKS"] if hooks else []), "-c", src, "-o", obj]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{res.stderr}")
        return obj, res.stderr

    srcs = sources()
    jobs = [(src, False) for src in srcs] + [(src, True) for src in srcs
                                             if os.path.basename(src) in TEST_HOOK_SOURCES]
    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        results = list(ex.map(compile_one, jobs))
    log = "".join(r[1] for r, (_, hooks) in zip(results, jobs) if not hooks)
    with open(os.path.join(BUILD, "ptxas.log"), "w") as f:
        f.write(log)
    if verbose:
        print(log)
    product = [r[0] for r, (_, hooks) in zip(results, jobs) if not hooks]
    hooked = {os.path.basename(src): r[0] for r, (src, hooks) in zip(results, jobs) if hooks}
    test_objs = [hooked.get(os.path.basename(src), obj) for src, obj in zip(srcs, product)]
    for objs, lib in ((product, LIB), (test_objs, TEST_LIB)):
        tmp = lib + f".tmp{os.getpid()}"
        subprocess.check_call(["nvcc", "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *objs, "-o", tmp])
        os.replace(tmp, lib)
    tmp = CEIL_LIB + f".tmp{os.getpid()}"
    res = subprocess.run(["nvcc", *NVCC_FLAGS, "-shared", CEIL_SRC, "-o", tmp], capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed for {CEIL_SRC}:\n{res.stderr}")
    os.replace(tmp, CEIL_LIB)
    return LIB
