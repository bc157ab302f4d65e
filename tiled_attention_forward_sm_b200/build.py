"""Build the sm_100a shared library ``libattn_b200.so`` in place.

    python -m tiled_attention_forward_sm_b200.build [--verbose] [--trace]

``--test-hooks`` builds ``libattn_b200_testhooks.so``: the attention and FP8
entry points compiled with ATTN_TEST_HOOKS, which adds
``int attn_test_set_hooks(unsigned long long wait_limit_ns, int withhold_load)``
(a shorter bounded-wait limit and one K/V load that CTA 0 skips, so that a
wait runs out and the kernels' abort path runs; see the GPU test of the
abort path).  The product library never carries these hooks.

``--checked`` builds ``libattn_b200_checked.so``: the same entry points as
the test-hooks library compiled with ATTN_BOUNDS_CHECKS as well, so that
every tensor-map coordinate and every O / LSE store index is checked against
the launch's tensor extents before the access (a failed check writes
ATTN_ERR_DEVICE_BOUNDS to the status word and skips the access), plus
``int attn_test_set_bad_kv_head(int offset)`` to plant one bad K/V head
index that the check must catch.  A debugging build; the product library
carries neither the checks nor the hook.

``--trace`` builds the timeline-tracing library ``libattn_b200_trace.so``
instead: the attention kernel compiled with its clock64 stamps at every role
hand-off (ATTN_TRACE_ENABLED) and the extra entry point
``int attn_trace_set_buffer(void* dev_buf)``.  It is a debugging build, read
by ``tiled_attention_forward_sm_b200.trace``; the product library never
carries the stamps.

Runs nvcc for ``-gencode arch=compute_100a,code=sm_100a`` with line info; the
library is written beside this file so it travels with the source tree.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libattn_b200.so")
TRACE_LIB = os.path.join(PKG, "libattn_b200_trace.so")
TEST_HOOKS_LIB = os.path.join(PKG, "libattn_b200_testhooks.so")
CHECKED_LIB = os.path.join(PKG, "libattn_b200_checked.so")
SOURCES = [os.path.join(CSRC, f) for f in ("attn_fwd.cu", "fp8.cu", "fp4.cu", "kmeans.cu", "pair.cu",
                                           "host_io.cu")]
HEADERS = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))] + [
    os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    f"-I{INCLUDE}",
]


def nvcc_path() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    cmd = [nvcc_path(), *NVCC_FLAGS, *(["-Xptxas", "-v"] if verbose else []), "-o", LIB, *SOURCES]
    subprocess.check_call(cmd)
    return LIB


def build_trace(force: bool = False, verbose: bool = False) -> str:
    """The tracing library (attention entry points of attn_fwd.cu only)."""
    src = os.path.join(CSRC, "attn_fwd.cu")
    if (not force and os.path.exists(TRACE_LIB) and
            all(os.path.getmtime(p) <= os.path.getmtime(TRACE_LIB) for p in [src] + HEADERS)):
        return TRACE_LIB
    cmd = [nvcc_path(), *NVCC_FLAGS, "-DATTN_TRACE_ENABLED", *(["-Xptxas", "-v"] if verbose else []),
           "-o", TRACE_LIB, src]
    subprocess.check_call(cmd)
    return TRACE_LIB


def build_test_hooks(force: bool = False) -> str:
    """The test-hooks library (attention and FP8 entry points)."""
    srcs = [os.path.join(CSRC, f) for f in ("attn_fwd.cu", "fp8.cu")]
    if (not force and os.path.exists(TEST_HOOKS_LIB) and
            all(os.path.getmtime(p) <= os.path.getmtime(TEST_HOOKS_LIB) for p in srcs + HEADERS)):
        return TEST_HOOKS_LIB
    cmd = [nvcc_path(), *NVCC_FLAGS, "-DATTN_TEST_HOOKS", "-o", TEST_HOOKS_LIB, *srcs]
    subprocess.check_call(cmd)
    return TEST_HOOKS_LIB


def build_checked(force: bool = False) -> str:
    """The bounds-checked test library (attention and FP8 entry points)."""
    srcs = [os.path.join(CSRC, f) for f in ("attn_fwd.cu", "fp8.cu")]
    if (not force and os.path.exists(CHECKED_LIB) and
            all(os.path.getmtime(p) <= os.path.getmtime(CHECKED_LIB) for p in srcs + HEADERS)):
        return CHECKED_LIB
    cmd = [nvcc_path(), *NVCC_FLAGS, "-DATTN_TEST_HOOKS", "-DATTN_BOUNDS_CHECKS", "-o",
           CHECKED_LIB, *srcs]
    subprocess.check_call(cmd)
    return CHECKED_LIB


if __name__ == "__main__":
    if "--test-hooks" in sys.argv:
        print(build_test_hooks(force=True))
    elif "--checked" in sys.argv:
        print(build_checked(force=True))
    elif "--trace" in sys.argv:
        print(build_trace(force=True, verbose="--verbose" in sys.argv))
    else:
        build(force=True, verbose="--verbose" in sys.argv)
        print(LIB)
