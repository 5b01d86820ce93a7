"""Build libdz.so (the C-ABI library) in-tree for sm_100a with nvcc.

Also builds libdz_test.so from the same sources for the tests: every bounded
device wait gives up after 20 ms instead of 2 s; every kernel checks its global
indexes against the extents of their buffers (DZ_DEBUG_BOUNDS: a failed check skips
the access and records DZ_ERR_BOUNDS in the status word); and the library exports
test-only calls: dz_test_fill_split_counters (presets the split counters so that a
merge's wait can never complete), dz_test_shrink_out (understates the attention
output's extent), dz_test_bounds_faults (index faults counted on the host) and
dz_test_plan_schedule (the attention work split).  Nothing but the tests loads it.

Usage: python -m causal_video_diffusion_rope_b200.build [--verbose-ptxas]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libdz.so")
TEST_LIB = os.path.join(HERE, "libdz_test.so")
TEST_DEFINES = ["-DDZ_TEST_HOOKS", "-DDZ_DEBUG_BOUNDS", "-DDZ_WAIT_NS=20000000ull"]
SOURCES = ["dz_api.cu", "dz_kernels.cu", "dz_attn.cu", "dz_qkv.cu", "dz_bwd.cu"]
HEADERS = ["dz_internal.cuh", "dz_ops.cuh", "dz_ptx.cuh"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "dz.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(out: str, defines, verbose_ptxas: bool) -> None:
    cmd = [
        nvcc_path(), "-O3", "-std=c++17", "-lineinfo",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-Xcompiler", "-fPIC", "-shared",
        "-I", os.path.join(ROOT, "include"),
        "-o", out + ".tmp",
    ] + list(defines)
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose_ptxas:
        sys.stderr.write(res.stderr)
    os.replace(out + ".tmp", out)


def build(force: bool = False, verbose_ptxas: bool = False, test_lib: bool = True) -> str:
    """Compile libdz.so (and, unless test_lib is False, libdz_test.so) if stale or forced."""
    if force or _stale(LIB):
        _compile(LIB, [], verbose_ptxas)
    if test_lib and (force or _stale(TEST_LIB)):
        _compile(TEST_LIB, TEST_DEFINES, False)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv))
